// Status codes, thread-local error messages and small device queries.
#include <cstdarg>
#include <cstring>
#include <mutex>
#include <vector>

#include "sf_internal.h"

namespace sf {

static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

sf_status fail(sf_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  set_error(buf);
  return st;
}

sf_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SF_ECUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

int sm_count() {
  static std::mutex mu;
  static std::vector<int> counts;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(counts.size()) <= dev) counts.resize(dev + 1, 0);
  if (counts[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    counts[dev] = n;
  }
  return counts[dev];
}

}  // namespace sf

extern "C" {

const char* sf_version(void) { return "sf 0.1 (sm_100a)"; }

const char* sf_status_string(sf_status s) {
  switch (s) {
    case SF_OK: return "SF_OK";
    case SF_EINVAL: return "SF_EINVAL";
    case SF_ENOMEM: return "SF_ENOMEM";
    case SF_ECUDA: return "SF_ECUDA";
    case SF_ETIMEOUT: return "SF_ETIMEOUT";
    case SF_ENOTIMPL: return "SF_ENOTIMPL";
  }
  return "SF_UNKNOWN";
}

size_t sf_last_error(char* buf, size_t len) {
  const std::string& m = sf::g_last_error;
  if (buf && len) {
    size_t n = m.size() < len - 1 ? m.size() : len - 1;
    memcpy(buf, m.data(), n);
    buf[n] = '\0';
  }
  return m.size();
}

}  // extern "C"
