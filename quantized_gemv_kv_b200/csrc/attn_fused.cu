// sf_attn_decode_refine as one kernel: a thread-block cluster per KV group
// runs the whole refined decode attention of the group on chip.
//
// The pass structure is that of the multi-kernel pipeline (attn.cu) -- fast
// resident scores, the exact top-k per query head through a proven error
// band, refined scores and values for the union of the group's selections,
// softmax and output -- but the intermediate results never leave the
// cluster.  Each CTA of the cluster owns a contiguous token range of the
// group:
//
//   1  score    stream the range's 2-bit keys through per-warp cp.async
//               rings into integer tensor-core MMAs; the fast scores of all
//               the group's heads stay in shared memory.
//   2  tau      the k-th largest fast score per head is bracketed by radix
//               levels over the order-preserving score keys: every CTA builds
//               a histogram of its own scores, the cluster barrier publishes
//               them, and every CTA sums all of them through distributed
//               shared memory and picks the bin that holds the k-th largest.
//               The first level's 256 bins cover the 4 binades below the
//               group's maximum (1/64 binade each); a level stops once the
//               chosen bin is small.  The bracket [tau_lo, tau_hi] replaces
//               the exact tau of the multi-kernel pipeline: a token whose fast
//               score exceeds tau_hi + 2 eps is in the top k outright, one
//               below tau_lo - 2 eps is out, and the band in between is
//               re-keyed exactly and ranked.
//   3  rank     the CTA that owns a token re-keys it exactly (fp64 / integer
//               dot products, as in the pipeline) and pushes (key, token) to
//               the shared memory of the head's owner CTA, which ranks the
//               band (key desc, token asc) and sets the winners' bits in the
//               token bitmask of the CTA that holds each token.
//   4  output   per CTA: refined scores for its union tokens, softmax
//               weights against the CTA's maximum (written in place over the
//               scores), the value MMAs over the L2-resident value codes, the
//               refined value corrections; then the cluster merges the CTAs'
//               (max, sum, output) through distributed shared memory.
//
// Scratch is shared memory, except the overflow lists of a band too large for
// its owner's shared memory, which go to the caller's workspace.  No
// spin-waits: all cross-CTA ordering is the cluster barrier.
#include <cooperative_groups.h>

#include <mutex>

#include "attn_common.cuh"

namespace {

namespace cg = cooperative_groups;

constexpr int kFThreads = 256;
constexpr int kFW = kFThreads / 32;   // warps per CTA
constexpr int kFMaxCluster = 16;      // CTAs per KV group (non-portable cluster size)
constexpr int kFRing = 4;             // cp.async stages per warp, one 16-token tile each
constexpr int kFBins = 256;           // bins of a radix level's window
constexpr int kFFirstShift = 17;      // first window: 256 bins of 2^17 keys = 1/64 binade each
constexpr int kFStop = 48;            // a chosen bin this small ends the levels
constexpr int kFMaxLevels = 8;
constexpr int kFBandCap = kFThreads;  // band entries per head ranked in the owner's shared memory
constexpr int kFStgCap = 128;         // union tokens per CTA whose value refinement rows are staged
constexpr int kFLocalBand = 256;      // band entries of one CTA listed in shared memory

__host__ __device__ constexpr int fused_rmax(int grp) { return grp <= 4 ? 2048 : 1024; }
__host__ __device__ constexpr int fused_nt(int grp) { return 2 * grp <= 8 ? 1 : 2; }

// Dynamic shared memory of one CTA owning R tokens (R a multiple of 32).
struct FusedSmem {
  int sc;     // fp32 scores [GRP][R]; then the f16 weight tile [8 NT][R + 8]; then the per-warp output tiles
  int ring;   // [kFW][kFRing][16 rows][8 words]: key codes, later value codes
  int ksz;    // [R] key scale | zero << 16
  int vsz;    // [R] value scale | zero << 16
  int hist;   // [2][GRP][kFBins] this CTA's level histograms (double-buffered)
  int hsum;   // [GRP][kFBins] the cluster's sum of the current level
  int hred;   // [GRP][kFBins] (this CTA's slice of) the cluster's sum, read remotely
  int bkey;   // [kFBandCap] exact keys of the band of the head this CTA owns
  int btok;   // [kFBandCap] their tokens
  int stg;    // [kFStgCap][8 words] value refinement rows of union tokens
  int umask;  // [R / 32] token bitmask of the group's union over this range
  int ulist;  // [R] union tokens of this range, ascending (u16 local index)
  int total;
};

__host__ __device__ inline FusedSmem fused_smem(int grp, int R) {
  FusedSmem s{};
  int off = 0;
  auto take = [&](int bytes) {
    const int o = off;
    off = (off + bytes + 15) & ~15;
    return o;
  };
  const int nt = fused_nt(grp);
  int scb = grp * R * 4;
  scb = scb > nt * 8 * (R + 8) * 2 ? scb : nt * 8 * (R + 8) * 2;
  scb = scb > kFW * grp * D * 4 ? scb : kFW * grp * D * 4;
  s.sc = take(scb);
  s.ring = take(kFW * kFRing * 16 * kWordsPerRow * 4);
  s.ksz = take(R * 4);
  s.vsz = take(R * 4);
  s.hist = take(2 * grp * kFBins * 4);
  s.hsum = take(grp * kFBins * 4);
  s.hred = take(grp * kFBins * 4);
  s.bkey = take(kFBandCap * 8);
  s.btok = take(kFBandCap * 4);
  s.stg = take(kFStgCap * kWordsPerRow * 4);
  s.umask = take(R / 32 * 4);
  s.ulist = take(R * 2);
  s.total = off;
  return s;
}

struct FusedArgs {
  const uint16_t* q;
  const uint32_t* k_res;
  const uint32_t* k_ref;
  const uint32_t* v_res;
  const uint32_t* v_ref;
  const uint16_t* k_scale;
  const uint16_t* k_zero;
  const uint16_t* v_scale;
  const uint16_t* v_zero;
  int T, k, R;
  int S;              // rows per KV head in the K/V arrays (the cache's stride)
  int32_t* sel_out;
  int32_t* sel_n;
  float* out;
  // caller workspace, touched only by a band larger than kFBandCap
  double* ovf_key;   // [Hq][T]
  int32_t* ovf_tok;  // [Hq][T]
  int32_t* ovf_sel;  // [Hq][k]
  // caller workspace: the CTAs' (max, sum, output) partials and union counts
  float* gpart;      // [Hkv][16][GRP][D + 2]
  int32_t* gcnt;     // [Hkv][16]
};


// Distributed shared memory: the address of p in CTA `rank` of the cluster,
// and plain (relaxed) accesses to it; the cluster barrier orders them.
__device__ __forceinline__ uint32_t dsm_addr(const void* p, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(r)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t dsm_ld_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ int4 dsm_ld_v4(uint32_t a) {
  int4 v;
  asm volatile("ld.shared::cluster.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a)
               : "memory");
  return v;
}
__device__ __forceinline__ void dsm_st_f64(uint32_t a, double v) {
  asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(a), "d"(v) : "memory");
}
__device__ __forceinline__ void dsm_st_u32(uint32_t a, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t dsm_atom_add(uint32_t a, uint32_t v) {
  uint32_t old;
  asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(a), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void dsm_red_or(uint32_t a, uint32_t v) {
  asm volatile("red.shared::cluster.or.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// frexp exponent of a nonzero finite float (v = m 2^e, 0.5 <= |m| < 1).
__device__ __forceinline__ int fexp(float v) {
  const uint32_t b = __float_as_uint(v) & 0x7FFFFFFFu;
  const int ef = static_cast<int>(b >> 23);
  return ef ? ef - 126 : -117 - static_cast<int>(__clz(b));
}
// 2^k as a float for -149 <= k <= 127.
__device__ __forceinline__ float pow2f(int k) {
  return k >= -126 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23) : __uint_as_float(1u << (k + 149));
}
// v 2^k (exact unless the result leaves the normal range), -149 <= k <= 254.
__device__ __forceinline__ float scale2(float v, int k) {
  return k <= 127 ? v * pow2f(k) : (v * pow2f(k - 127)) * pow2f(127);
}

// Exact int -> fp32 for |v| < 2^22 on the integer and FP32 pipes (no
// conversion instruction): v rides in the mantissa of 1.5 * 2^23.
__device__ __forceinline__ float i2f_exact(int v) { return __int_as_float(0x4B400000 + v) - 12582912.0f; }

// Smallest s >= 0 with width <= 256 << s.
__device__ __forceinline__ int level_shift(unsigned long long width) {
  int s = 0;
  while ((static_cast<unsigned long long>(kFBins) << s) < width) ++s;
  return s;
}

// The exact key of one token for head h (the multi-kernel pipeline's
// definition): integer byte-plane dot products when the head's q spans at most
// 15 binades, else fp64 fmas.
__device__ __forceinline__ double exact_key(const uint32_t* w, double sv, double z, bool int_keys,
                                           const uint32_t (*qpl)[8][4], long long qxsum, int qe, const float* qf) {
  if (int_keys) {
    unsigned d0 = 0, d1 = 0;
    int d2 = 0;
#pragma unroll
    for (int wi = 0; wi < 8; ++wi)
#pragma unroll
      for (int kq = 0; kq < 4; ++kq) {
        const unsigned c = (w[wi] >> (2 * kq)) & 0x03030303u;
        d0 = __dp4a(c, qpl[0][wi][kq], d0);
        d1 = __dp4a(c, qpl[1][wi][kq], d1);
        d2 = __dp4a(static_cast<int>(c), static_cast<int>(qpl[2][wi][kq]), d2);
      }
    const long long P = static_cast<long long>(d0) + 256ll * d1 + 65536ll * d2;
    const double cq = ldexp(static_cast<double>(P), qe - 23);
    const double qsum = ldexp(static_cast<double>(qxsum), qe - 23);
    return sv * fma(1.5 - z, qsum, 4.0 * cq);
  }
  double E[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int wi = 0; wi < 8; ++wi) {
    const uint32_t word = w[wi];
#pragma unroll 1
    for (int jj = 0; jj < 4; ++jj)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = 4 * jj + u;
        const double c = static_cast<double>((word >> (2 * j)) & 3u);
        E[u] = fma(static_cast<double>(qf[16 * wi + j]), c * 4.0 + 1.5 - z, E[u]);
      }
  }
  return sv * ((E[0] + E[1]) + (E[2] + E[3]));
}

// Warp search of a level's 256 summed bins from the top for the kk-th
// largest: returns the bin (or -1 when it lies below the window), the count
// above that bin, and the window's total.  Lane l holds the run of bins
// [248 - 8 l, 256 - 8 l); one scan over the lanes finds the run that crosses
// kk, and that lane walks it.
__device__ __forceinline__ void window_find(const int* hs, int kk, int* bin_out, int* above_out, int* tot_out) {
  const int lane = threadIdx.x & 31;
  const int4* h4 = reinterpret_cast<const int4*>(hs + kFBins - 8 - 8 * lane);
  const int4 lo4 = h4[0], hi4 = h4[1];
  const int c[8] = {hi4.w, hi4.z, hi4.y, hi4.x, lo4.w, lo4.z, lo4.y, lo4.x};  // descending bins
  int sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) sum += c[j];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int excl = incl - sum, tot = __shfl_sync(0xffffffffu, incl, 31);
  const unsigned m = __ballot_sync(0xffffffffu, excl < kk && incl >= kk);
  int bin = -1, above = tot;
  if (m) {
    const int src = __ffs(m) - 1;
    int b = 0, a = 0;
    if (lane == src) {
      a = excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (a + c[j] >= kk) {
          b = kFBins - 1 - 8 * lane - j;
          break;
        }
        a += c[j];
      }
    }
    bin = __shfl_sync(0xffffffffu, b, src);
    above = __shfl_sync(0xffffffffu, a, src);
  }
  *bin_out = bin;
  *above_out = above;
  *tot_out = tot;
}

// 12-pass radix selection over (exact key desc, token asc) of n entries in
// global memory: the kk winners go to sel.  Only for a band that did not fit
// its owner's shared memory.  All threads call.
__device__ __noinline__ void rank_select_global(const double* __restrict__ key, const int32_t* __restrict__ tok, int n, int kk,
                                   int* hist, int* scan_scratch, int* binfo, int32_t* __restrict__ sel) {
  const int tid = threadIdx.x;
  // composite 96-bit key: okey64(key) then ~token, both descending
  unsigned long long pk = 0, mk = 0;
  uint32_t pt = 0, mt = 0;
  int kr = kk;
  for (int pass = 0; pass < 12; ++pass) {
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += blockDim.x) {
      const unsigned long long a = okey64(key[i]);
      const uint32_t b = ~static_cast<uint32_t>(tok[i]);
      if ((a & mk) != pk || (b & mt) != pt) continue;
      const int digit = pass < 8 ? static_cast<int>((a >> (56 - 8 * pass)) & 255u)
                                 : static_cast<int>((b >> (24 - 8 * (pass - 8))) & 255u);
      atomicAdd(&hist[digit], 1);
    }
    __syncthreads();
    find_bin_from_top_block(hist, 256, kr, binfo, scan_scratch);
    if (pass < 8) {
      pk |= static_cast<unsigned long long>(binfo[0]) << (56 - 8 * pass);
      mk |= 255ull << (56 - 8 * pass);
    } else {
      pt |= static_cast<uint32_t>(binfo[0]) << (24 - 8 * (pass - 8));
      mt |= 255u << (24 - 8 * (pass - 8));
    }
    kr = binfo[1];
    __syncthreads();
  }
  // the composite keys are distinct; the winners are those >= the kk-th
  int cnt = 0;
  for (int i = tid; i < n; i += blockDim.x) {
    const unsigned long long a = okey64(key[i]);
    const uint32_t b = ~static_cast<uint32_t>(tok[i]);
    cnt += (a > pk || (a == pk && b >= pt)) ? 1 : 0;
  }
  int tot;
  int pos = sfd::block_exclusive_scan(cnt, scan_scratch, &tot);
  for (int i = tid; i < n; i += blockDim.x) {
    const unsigned long long a = okey64(key[i]);
    const uint32_t b = ~static_cast<uint32_t>(tok[i]);
    if (a > pk || (a == pk && b >= pt)) sel[pos++] = tok[i];
  }
  __syncthreads();
}

// Re-keys one token of this CTA's range exactly for one head and pushes
// (key, token) to the band list of the head's owner; a full list spills to the
// workspace.  Rare (only tokens inside the error band of tau), so kept out of
// line.
__device__ __noinline__ void band_push(const uint32_t* __restrict__ krow, uint32_t kz, bool int_keys,
                                       const uint32_t (*qpl)[8][4], long long qxsum, int qe, const float* qf,
                                       int owner, int* bcnt, double* bkey, int* btok, double* __restrict__ ovf_key,
                                       int32_t* __restrict__ ovf_tok, int token) {
  const uint4* w4 = reinterpret_cast<const uint4*>(krow);
  const uint4 x0 = w4[0], x1 = w4[1];
  const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
  const double sv = static_cast<double>(sfd::half_bits_to_float(static_cast<uint16_t>(kz & 0xFFFFu)));
  const double z = static_cast<double>(sfd::half_bits_to_float(static_cast<uint16_t>(kz >> 16)));
  const double key = exact_key(w, sv, z, int_keys, qpl, qxsum, qe, qf);
  const uint32_t slot = dsm_atom_add(dsm_addr(bcnt, owner), 1u);
  if (slot < static_cast<uint32_t>(kFBandCap)) {
    dsm_st_f64(dsm_addr(bkey + slot, owner), key);
    dsm_st_u32(dsm_addr(btok + slot, owner), static_cast<uint32_t>(token));
  } else {
    ovf_key[slot] = key;
    ovf_tok[slot] = token;
  }
}

// Ranks a band that overflowed its owner's shared memory: the shared part is
// appended to the workspace list and the whole list is radix-selected there.
__device__ __noinline__ void rank_overflow(const double* bkey, const int* btok, int nb, int kB,
                                           double* __restrict__ gk, int32_t* __restrict__ gt,
                                           int32_t* __restrict__ sel, int* rhist, int* scan_scratch, int* binfo) {
  for (int i = threadIdx.x; i < kFBandCap; i += blockDim.x) {
    gk[i] = bkey[i];
    gt[i] = btok[i];
  }
  __syncthreads();
  rank_select_global(gk, gt, nb, kB, rhist, scan_scratch, binfo, sel);
}

template <int GRP>
__global__ void __launch_bounds__(kFThreads, 2) attn_fused_kernel(const FusedArgs a) {
  constexpr int NT = fused_nt(GRP);
  constexpr int kPT = fused_rmax(GRP) / kFThreads;  // tokens per thread in the per-token passes
  cg::cluster_group cl = cg::this_cluster();
  const int C = static_cast<int>(cl.num_blocks());
  const int r = static_cast<int>(cl.block_rank());
  const int g = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g8 = lane >> 2, tig = lane & 3;
  const int T = a.T, R = a.R, k = a.k;
  const int t0 = r * R;
  const int n = max(0, min(R, T - t0));  // tokens of this CTA: [t0, t0 + n)
  const int ntile = (n + 15) >> 4;
  const size_t row0 = static_cast<size_t>(g) * a.S + t0;
  const int kStr = R + 8;  // halves per weight row: conflict-free fragment loads
  const FusedSmem S = fused_smem(GRP, R);
  extern __shared__ __align__(16) unsigned char smem[];
  float* sc = reinterpret_cast<float*>(smem + S.sc);
  __half* as = reinterpret_cast<__half*>(smem + S.sc);
  uint32_t* ring = reinterpret_cast<uint32_t*>(smem + S.ring);
  uint32_t* ksz = reinterpret_cast<uint32_t*>(smem + S.ksz);
  uint32_t* vsz = reinterpret_cast<uint32_t*>(smem + S.vsz);
  int* hist = reinterpret_cast<int*>(smem + S.hist);
  int* hsum = reinterpret_cast<int*>(smem + S.hsum);
  int* hred = reinterpret_cast<int*>(smem + S.hred);
  double* bkey = reinterpret_cast<double*>(smem + S.bkey);
  int* btok = reinterpret_cast<int*>(smem + S.btok);
  uint32_t* stg = reinterpret_cast<uint32_t*>(smem + S.stg);
  uint32_t* umask = reinterpret_cast<uint32_t*>(smem + S.umask);
  uint16_t* ulist = reinterpret_cast<uint16_t*>(smem + S.ulist);
  // staging of the outright selections' key rows in the histograms' space
  // (after the radix levels): a slot per local token (0xFF: none), then the
  // rows, 16 words each (resident codes, refinement codes)
  uint8_t* smap = smem + S.hist;
  uint32_t* kst = reinterpret_cast<uint32_t*>(smem + S.hist + R);
  const int kst_cap = min(255, (S.hred - S.hist - R) / (2 * kWordsPerRow * 4));

  __shared__ int qx[GRP][D];         // fixed-point query heads
  __shared__ float qs[GRP][D];       // query heads in fp32 (exact: bf16)
  __shared__ float qsc[GRP], qsm[GRP];
  __shared__ uint32_t qpl[GRP][3][8][4];  // byte planes of qx in code-extraction order
  __shared__ uint32_t bfr[24][32];        // B fragments of qx, per lane
  __shared__ long long qxs[GRP];
  __shared__ int qe_sh[GRP], ikey_sh[GRP];
  __shared__ double l1_sh[GRP], eps_sh[GRP], hiA_sh[GRP];
  __shared__ float fthr_sh[GRP];
  __shared__ int flag_sh;
  __shared__ uint32_t l0[2 * GRP + 1];   // published: max key and min key per head, max key scale
  __shared__ uint32_t gl0[2 * GRP + 1];  // their cluster-wide values
  __shared__ uint32_t lo_sh[GRP], hi_sh[GRP], wlo_sh[GRP];  // key bracket of tau and the level's window
  __shared__ int s_sh[GRP], kk_sh[GRP], cnt_sh[GRP], done_sh[GRP];
  __shared__ int nal[GRP];               // published: tokens of this range selected outright, per head
  __shared__ int bcnt;                   // band entries pushed to this CTA (the owner of head r)
  __shared__ int lbn;                    // band entries of this range
  __shared__ int nst;                    // staged key rows
  __shared__ int lband[kFLocalBand];     // (token << 3 | head) of this range's band entries
  __shared__ int kB_sh;
  __shared__ int ucnt, uoff;             // union tokens of this range, and their offset in the group's list
  __shared__ float Fc[GRP][kFMaxCluster];
  __shared__ float Lh[GRP], Msh[GRP];
  __shared__ float red[kFW][GRP];
  __shared__ float red2[kFW][3 * GRP];
  __shared__ int scan_scratch[64];
  __shared__ int binfo[2];
  __shared__ int rhist[256];

  // ---- prologue: key ring, scales, q
  const int tpw = (ntile + kFW - 1) / kFW;
  const int tile0 = min(ntile, warp * tpw), tile1 = min(ntile, tile0 + tpw);
  auto issue = [&](const uint32_t* src, int ti) {
    const int st = (ti - tile0) % kFRing;
    const int row = 16 * ti + (lane >> 1);
    if (row < n)
      cp_async16_attn(ring + ((warp * kFRing + st) * 16 + (lane >> 1)) * kWordsPerRow + (lane & 1) * 4,
                      src + (row0 + row) * kWordsPerRow + (lane & 1) * 4);
  };
  for (int i = 0; i < kFRing - 2; ++i) {  // two tiles in flight, two being scored
    if (tile0 + i < tile1) issue(a.k_res, tile0 + i);
    cp_async_commit_attn();
  }
  if (tid < GRP) {
    l0[tid] = 0u;
    l0[GRP + tid] = 0xFFFFFFFFu;
    nal[tid] = 0;
  }
  if (tid == 0) {
    l0[2 * GRP] = 0u;
    bcnt = 0;
    lbn = 0;
    nst = 0;
    flag_sh = 0;
  }
  {
    // every load of this thread is issued before the first store; the key
    // scales' maximum (for the error bound) comes along
    uint32_t kzv[kPT], vzv[kPT];
#pragma unroll
    for (int j = 0; j < kPT; ++j) {
      const int i = tid + j * kFThreads;
      kzv[j] = vzv[j] = 0u;
      if (i < n) {
        kzv[j] = static_cast<uint32_t>(a.k_scale[row0 + i]) | (static_cast<uint32_t>(a.k_zero[row0 + i]) << 16);
        vzv[j] = static_cast<uint32_t>(a.v_scale[row0 + i]) | (static_cast<uint32_t>(a.v_zero[row0 + i]) << 16);
      }
    }
    float smx = 0.0f;
#pragma unroll
    for (int j = 0; j < kPT; ++j) {
      const int i = tid + j * kFThreads;
      if (i < n) {
        ksz[i] = kzv[j];
        vsz[i] = vzv[j];
        smx = fmaxf(smx, sfd::half_bits_to_float(static_cast<uint16_t>(kzv[j] & 0xFFFFu)));
      }
    }
    smx = warp_max(smx);
    __syncthreads();  // l0 is initialised
    if (lane == 0) atomicMax(&l0[2 * GRP], __float_as_uint(smx));
  }
  for (int i = tid; i < R / 32; i += kFThreads) umask[i] = 0u;
  // query heads: warp h builds head h (4 dims per lane)
  for (int h = warp; h < GRP; h += kFW) {
    float v[4];
    float am = 0.0f;
    double l1 = 0.0;
    int emin = 100000, emax = -100000;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[i] = sfd::bf16_bits_to_float(a.q[(static_cast<size_t>(g) * GRP + h) * D + 4 * lane + i]);
      qs[h][4 * lane + i] = v[i];
      am = fmaxf(am, fabsf(v[i]));
      l1 += fabs(static_cast<double>(v[i]));
      if (v[i] != 0.0f) {
        const int e = fexp(v[i]);
        emin = min(emin, e);
        emax = max(emax, e);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      emin = min(emin, __shfl_xor_sync(0xffffffffu, emin, o));
      emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
    }
    // the sum of q (any order: the error bound covers it), the exponent of
    // max |q| (the largest exponent)
    float qsum_l = (v[0] + v[1]) + (v[2] + v[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qsum_l += __shfl_xor_sync(0xffffffffu, qsum_l, o);
    const int e = emax >= emin ? emax : 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) qx[h][4 * lane + i] = __float2int_rn(scale2(v[i], 23 - e));
    if (lane == 0) {
      const int span = emax >= emin ? emax - emin : 0;  // binades spanned by the nonzero q
      qsc[h] = pow2f(e - 23);
      qsm[h] = qsum_l;
      qe_sh[h] = e;
      ikey_sh[h] = span <= 15;
      l1_sh[h] = l1;
      // 53 - 9 - b - log2(d) with b = 4, d = 128: beyond it the exact key is not exact
      if (span > 53 - 9 - 4 - 7) atomicOr(&flag_sh, 1);
    }
  }
  __syncthreads();
  for (int e = tid; e < GRP * 96; e += kFThreads) {
    const int h = e / 96, x = e % 96, p = x / 32, wi = (x / 4) & 7, kq = x & 3;
    uint32_t v = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) v |= ((static_cast<uint32_t>(qx[h][16 * wi + kq + 4 * b]) >> (8 * p)) & 0xFFu) << (8 * b);
    qpl[h][p][wi][kq] = v;
  }
  for (int h = warp; h < GRP; h += kFW) {
    long long sx = static_cast<long long>(qx[h][lane]) + qx[h][lane + 32] + qx[h][lane + 64] + qx[h][lane + 96];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sx += __shfl_xor_sync(0xffffffffu, sx, o);
    if (lane == 0) qxs[h] = sx;
  }
  // B fragments (column n = g8 is query head g8, zero beyond the group),
  // built once per CTA: word [ks][p][half][lane]
  for (int e = tid; e < 24 * 32; e += kFThreads) {
    const int ln = e & 31, f = e >> 5, ks = f / 6, p = (f / 2) % 3, half = f & 1;
    const int gg = ln >> 2, tt = ln & 3;
    uint32_t v = 0;
    if (gg < GRP) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        v |= ((static_cast<uint32_t>(qx[gg][16 * (2 * ks + half) + tt + 4 * i]) >> (8 * p)) & 0xFFu) << (8 * i);
    }
    bfr[f][ln] = v;
  }
  __syncthreads();

  // ---- 1. fast scores of the range (integer tensor cores, keys from the ring)
  {
    uint32_t bq[4][3][2];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int p = 0; p < 3; ++p)
#pragma unroll
        for (int half = 0; half < 2; ++half) bq[ks][p][half] = bfr[(ks * 3 + p) * 2 + half][lane];
    // this lane's heads 2 tig, 2 tig + 1 (the epilogue runs on lanes holding a
    // head); with four heads, 2 (tig & 1) and the next, lanes tig >= 2 scoring
    // the second token of each tile (columns 4..7 of the MMA are padding)
    constexpr bool kSwap = GRP == 4;
    const int h0 = kSwap ? 2 * (tig & 1) : 2 * tig, h1 = h0 + 1;
    const bool on = h0 < GRP;
    const float qsc0 = on ? qsc[h0] : 0.0f, qsm0 = on ? qsm[h0] : 0.0f;
    const float qsc1 = h1 < GRP ? qsc[h1] : 0.0f, qsm1 = h1 < GRP ? qsm[h1] : 0.0f;
    for (int ti = tile0; ti < tile1; ti += 2) {
      if (ti + kFRing - 2 < tile1) issue(a.k_res, ti + kFRing - 2);
      cp_async_commit_attn();
      if (ti + kFRing - 1 < tile1) issue(a.k_res, ti + kFRing - 1);
      cp_async_commit_attn();
      cp_async_wait_attn<2>();
      __syncwarp();
      // two independent tiles: six accumulator chains interleave
      uint32_t wa[2][8], wb[2][8];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t* kr = ring + (warp * kFRing + (ti + u - tile0) % kFRing) * 16 * kWordsPerRow;
        const uint4* pa = reinterpret_cast<const uint4*>(kr + g8 * kWordsPerRow);
        const uint4* pb = reinterpret_cast<const uint4*>(kr + (g8 + 8) * kWordsPerRow);
        const uint4 xa0 = pa[0], xa1 = pa[1], xb0 = pb[0], xb1 = pb[1];
        wa[u][0] = xa0.x; wa[u][1] = xa0.y; wa[u][2] = xa0.z; wa[u][3] = xa0.w;
        wa[u][4] = xa1.x; wa[u][5] = xa1.y; wa[u][6] = xa1.z; wa[u][7] = xa1.w;
        wb[u][0] = xb0.x; wb[u][1] = xb0.y; wb[u][2] = xb0.z; wb[u][3] = xb0.w;
        wb[u][4] = xb1.x; wb[u][5] = xb1.y; wb[u][6] = xb1.z; wb[u][7] = xb1.w;
      }
      int d0[2][4], d1[2][4], d2[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i) d0[u][i] = d1[u][i] = d2[u][i] = 0;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const uint32_t a0 = (wa[u][2 * ks] >> (2 * tig)) & 0x03030303u;
          const uint32_t a1 = (wb[u][2 * ks] >> (2 * tig)) & 0x03030303u;
          const uint32_t a2 = (wa[u][2 * ks + 1] >> (2 * tig)) & 0x03030303u;
          const uint32_t a3 = (wb[u][2 * ks + 1] >> (2 * tig)) & 0x03030303u;
          mma_u8u8(d0[u], a0, a1, a2, a3, bq[ks][0][0], bq[ks][0][1]);
          mma_u8u8(d1[u], a0, a1, a2, a3, bq[ks][1][0], bq[ks][1][1]);
          mma_u8s8(d2[u], a0, a1, a2, a3, bq[ks][2][0], bq[ks][2][1]);
        }
      // d[u][i]: i = 0,1 -> token ta, heads 2 tig, 2 tig + 1; i = 2,3 -> token tb
      if constexpr (kSwap) {
        // lanes tig >= 2 take token tb of lane ^ 2 into slots 0, 1
        const bool up = tig >= 2;
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int i = 2; i < 4; ++i) {
            const int x0 = __shfl_xor_sync(0xffffffffu, d0[u][i], 2);
            const int x1 = __shfl_xor_sync(0xffffffffu, d1[u][i], 2);
            const int x2 = __shfl_xor_sync(0xffffffffu, d2[u][i], 2);
            if (up) {
              d0[u][i - 2] = x0;
              d1[u][i - 2] = x1;
              d2[u][i - 2] = x2;
            }
          }
      }
      if (on) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int ta = 16 * (ti + u) + g8, tb = ta + 8;
          const bool tv = ti + u < tile1;  // a missing second tile holds no keys
#pragma unroll
          for (int rr = 0; rr < (kSwap ? 1 : 2); ++rr) {
            const int tt = kSwap ? (tig >= 2 ? tb : ta) : (rr ? tb : ta);
            if (!tv || tt >= n) continue;
            const uint32_t kz = ksz[tt];
            const float sv = sfd::half_bits_to_float(static_cast<uint16_t>(kz & 0xFFFFu));
            const float zv = sfd::half_bits_to_float(static_cast<uint16_t>(kz >> 16));
            const int i0 = 2 * rr, i1 = 2 * rr + 1;
            // plane sums are below 2^17 in magnitude: exact conversions, the
            // same fp32 combination as the pipeline's score pass
            const float P0 =
                (i2f_exact(d2[u][i0]) * 65536.0f + i2f_exact(d1[u][i0]) * 256.0f + i2f_exact(d0[u][i0])) * qsc0;
            sc[h0 * R + tt] = (sv * fmaf(4.0f, P0, (1.5f - zv) * qsm0)) * kInvSqrtD;
            if (h1 < GRP) {
              const float P1 =
                  (i2f_exact(d2[u][i1]) * 65536.0f + i2f_exact(d1[u][i1]) * 256.0f + i2f_exact(d0[u][i1])) * qsc1;
              sc[h1 * R + tt] = (sv * fmaf(4.0f, P1, (1.5f - zv) * qsm1)) * kInvSqrtD;
            }
          }
        }
      }
      __syncwarp();  // the two stages are refilled by the next iteration's issues
    }
    cp_async_wait_attn<0>();
  }
  __syncthreads();
  // range extremes of the score keys per head
  {
    uint32_t kmx[GRP], kmn[GRP];
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      kmx[h] = 0u;
      kmn[h] = 0xFFFFFFFFu;
    }
    for (int i = tid; i < n; i += kFThreads)
#pragma unroll
      for (int h = 0; h < GRP; ++h) {
        const uint32_t key = okey32(sc[h * R + i]);
        kmx[h] = max(kmx[h], key);
        kmn[h] = min(kmn[h], key);
      }
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        kmx[h] = max(kmx[h], __shfl_xor_sync(0xffffffffu, kmx[h], o));
        kmn[h] = min(kmn[h], __shfl_xor_sync(0xffffffffu, kmn[h], o));
      }
      if (lane == 0) {
        atomicMax(&l0[h], kmx[h]);
        atomicMin(&l0[GRP + h], kmn[h]);
      }
    }
  }

  const bool selecting = k > 0 && k < T;
  if (selecting) {
    // ---- 2. bracket tau per head by radix levels over the cluster
    cl.sync();  // A: every CTA's extremes are published
    // two values per warp, 16 lanes each, lane c reading CTA c (whole warps
    // run every iteration: the shuffles need all their lanes)
    for (int jp = warp; jp < GRP + 1; jp += kFW) {
      const int j = 2 * jp + (lane >> 4), c = lane & 15;
      const bool valid = j < 2 * GRP + 1;
      const bool is_min = j >= GRP && j < 2 * GRP;
      uint32_t v = is_min ? 0xFFFFFFFFu : 0u;
      if (valid) v = c < C ? dsm_ld_u32(dsm_addr(&l0[j], c)) : l0[j];
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        const uint32_t y = __shfl_xor_sync(0xffffffffu, v, o);
        v = is_min ? min(v, y) : max(v, y);
      }
      if (valid && c == 0) gl0[j] = v;
    }
    __syncthreads();
    if (tid < GRP) {
      const float amax = fmaxf(fabsf(from_okey32(gl0[tid])), fabsf(from_okey32(gl0[GRP + tid])));
      eps_sh[tid] = select_eps(static_cast<double>(__uint_as_float(gl0[2 * GRP])), l1_sh[tid], qe_sh[tid], amax, 23);
      lo_sh[tid] = gl0[GRP + tid];
      hi_sh[tid] = gl0[tid];
      kk_sh[tid] = k;
      cnt_sh[tid] = T;
      done_sh[tid] = 0;
    }
    __syncthreads();
#pragma unroll 1
    for (int lev = 0; lev < kFMaxLevels; ++lev) {
      if (tid < GRP && !done_sh[tid]) {
        const unsigned long long width = static_cast<unsigned long long>(hi_sh[tid]) - lo_sh[tid] + 1ull;
        int s = level_shift(width);
        if (lev == 0 && s > kFFirstShift) s = kFFirstShift;
        const unsigned long long span = static_cast<unsigned long long>(kFBins) << s;
        wlo_sh[tid] = width > span ? static_cast<uint32_t>(hi_sh[tid] - (span - 1ull)) : lo_sh[tid];
        s_sh[tid] = s;
      }
      // this buffer was last read remotely two levels ago, before the previous
      // level's cluster barrier
      int* hb = hist + (lev & 1) * GRP * kFBins;
      for (int i = tid; i < GRP * kFBins; i += kFThreads) hb[i] = 0;
      __syncthreads();
      int ndone = 0;
#pragma unroll 1
      for (int h = 0; h < GRP; ++h) ndone += done_sh[h] != 0;
      if (ndone == GRP) break;  // uniform over the cluster: every CTA holds the same state
#pragma unroll 1
      for (int h = 0; h < GRP; ++h) {
        if (done_sh[h]) continue;
        const uint32_t wlo = wlo_sh[h], hi = hi_sh[h];
        const int s = s_sh[h];
        float v[kPT];  // every score of this thread is loaded before the first count
#pragma unroll
        for (int j = 0; j < kPT; ++j) {
          const int i = tid + j * kFThreads;
          v[j] = i < n ? sc[h * R + i] : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < kPT; ++j) {
          const uint32_t key = okey32(v[j]);
          if (tid + j * kFThreads < n && key >= wlo && key <= hi) atomicAdd(&hb[h * kFBins + ((key - wlo) >> s)], 1);
        }
      }
      cl.sync();  // B: every CTA's histogram of this level is published
      // the sum over the cluster in two steps: CTA r sums its slice of the
      // bins over every CTA, then every CTA gathers all the slices
      {
        constexpr int Q = GRP * kFBins / 4;  // int4s of a histogram
        const int S4 = (Q + C - 1) / C;
        for (int q = r * S4 + tid; q < min(Q, (r + 1) * S4); q += kFThreads) {
          int4 acc = make_int4(0, 0, 0, 0);
#pragma unroll 4
          for (int c = 0; c < C; ++c) {
            const int4 v = dsm_ld_v4(dsm_addr(reinterpret_cast<const int4*>(hb) + q, c));
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
          }
          reinterpret_cast<int4*>(hred)[q] = acc;
        }
        cl.sync();  // B2: every slice is summed
        for (int q = tid; q < Q; q += kFThreads)
          reinterpret_cast<int4*>(hsum)[q] = dsm_ld_v4(dsm_addr(reinterpret_cast<const int4*>(hred) + q, q / S4));
      }
      __syncthreads();
      if (warp < GRP && !done_sh[warp]) {
        int bin, above, tot;
        window_find(hsum + warp * kFBins, kk_sh[warp], &bin, &above, &tot);
        if (lane == 0) {
          const int s = s_sh[warp];
          const uint32_t wlo = wlo_sh[warp];
          if (bin < 0) {  // below the window: every window token ranks above
            hi_sh[warp] = wlo - 1u;
            kk_sh[warp] -= tot;
            cnt_sh[warp] -= tot;
          } else {
            const unsigned long long blo = static_cast<unsigned long long>(wlo) + (static_cast<unsigned long long>(bin) << s);
            const unsigned long long bhi = blo + (1ull << s) - 1ull;
            lo_sh[warp] = static_cast<uint32_t>(blo);
            hi_sh[warp] = static_cast<uint32_t>(bhi < hi_sh[warp] ? bhi : hi_sh[warp]);
            kk_sh[warp] -= above;
            cnt_sh[warp] = hsum[warp * kFBins + bin];
            if (cnt_sh[warp] <= kFStop || s == 0) done_sh[warp] = 1;
          }
        }
      }
      __syncthreads();
    }

    // ---- 3. outright selections and the band, re-keyed exactly and pushed
    //         to the head's owner (CTA h)
    if (tid < GRP) {
      hiA_sh[tid] = static_cast<double>(from_okey32(hi_sh[tid])) + 2.0 * eps_sh[tid];
      fthr_sh[tid] = __double2float_ru(static_cast<double>(from_okey32(lo_sh[tid])) - 2.0 * eps_sh[tid]);
    }
    // the histograms are dead (and no longer read remotely): their space
    // stages the key rows of the outright selections for the refined scores
    for (int w = tid; w < R / 4; w += kFThreads) reinterpret_cast<uint32_t*>(smap)[w] = 0xFFFFFFFFu;
    __syncthreads();
    // pass 1: the outright selections (bitmask, counts per head) and a list
    // of this range's band entries; pass 2 re-keys the entries in parallel
    {
      int nA[GRP];
#pragma unroll
      for (int h = 0; h < GRP; ++h) nA[h] = 0;
#pragma unroll
      for (int j = 0; j < kPT; ++j) {
        const int i = tid + j * kFThreads;
        if (i >= n) break;
        bool any = false;
#pragma unroll
        for (int h = 0; h < GRP; ++h) {
          const float v = sc[h * R + i];
          if (static_cast<double>(v) > hiA_sh[h]) {
            any = true;
            ++nA[h];
          } else if (v >= fthr_sh[h]) {
            const int pos = atomicAdd(&lbn, 1);
            if (pos < kFLocalBand) lband[pos] = (i << 3) | h;
          }
        }
        if (any) {
          atomicOr(&umask[i >> 5], 1u << (i & 31));
          const int s = atomicAdd(&nst, 1);
          if (s < kst_cap) {
            uint32_t* dst = kst + s * 2 * kWordsPerRow;
            const uint32_t* kr = a.k_res + (row0 + i) * kWordsPerRow;
            const uint32_t* kf = a.k_ref + (row0 + i) * kWordsPerRow;
            cp_async16_attn(dst, kr);
            cp_async16_attn(dst + 4, kr + 4);
            cp_async16_attn(dst + 8, kf);
            cp_async16_attn(dst + 12, kf + 4);
            smap[i] = static_cast<uint8_t>(s);
          }
        }
      }
#pragma unroll
      for (int h = 0; h < GRP; ++h) {
        int v = nA[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && v) atomicAdd(&nal[h], v);
      }
      cp_async_commit_attn();  // the staged key rows
    }
    __syncthreads();
    {
      const int nb = lbn;
      for (int e = tid; e < nb; e += kFThreads) {
        int i = 0, h = 0;
        if (nb <= kFLocalBand) {
          i = lband[e] >> 3;
          h = lband[e] & 7;
        } else {  // the list overflowed: the e-th band entry in (token, head) order is found again
          int cnt = 0;
          bool found = false;
          for (int ii = 0; ii < n && !found; ++ii)
            for (int hh = 0; hh < GRP && !found; ++hh) {
              const float v = sc[hh * R + ii];
              if (!(static_cast<double>(v) > hiA_sh[hh]) && v >= fthr_sh[hh] && cnt++ == e) {
                i = ii;
                h = hh;
                found = true;
              }
            }
        }
        band_push(a.k_res + (row0 + i) * kWordsPerRow, ksz[i], ikey_sh[h] != 0, qpl[h], qxs[h], qe_sh[h], qs[h], h,
                  &bcnt, bkey, btok, a.ovf_key + (static_cast<size_t>(g) * GRP + h) * T,
                  a.ovf_tok + (static_cast<size_t>(g) * GRP + h) * T, t0 + i);
      }
    }
    cl.sync();  // C: band entries and outright counts are published

    // ---- the owner of head h = r ranks its band: (key desc, token asc)
    if (r < GRP) {
      const int h = r;
      if (warp == 0) {
        int v = lane < C ? static_cast<int>(dsm_ld_u32(dsm_addr(&nal[h], lane))) : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) kB_sh = max(0, k - v);
      }
      __syncthreads();
      const int kB = kB_sh, nb = bcnt;
      if (nb <= kFBandCap) {
        if (tid < nb) {
          const unsigned long long ki = okey64(bkey[tid]);
          const int ti = btok[tid];
          int rank = 0;
#pragma unroll 4
          for (int j = 0; j < nb; ++j) {
            const unsigned long long kj = okey64(bkey[j]);
            rank += (kj > ki || (kj == ki && btok[j] < ti)) ? 1 : 0;
          }
          if (rank < kB) {
            const int c = ti / R, li = ti - c * R;
            dsm_red_or(dsm_addr(&umask[li >> 5], c), 1u << (li & 31));
          }
        }
      } else {
        const size_t base = (static_cast<size_t>(g) * GRP + h) * T;
        int32_t* sel = a.ovf_sel + (static_cast<size_t>(g) * GRP + h) * k;
        rank_overflow(bkey, btok, nb, kB, a.ovf_key + base, a.ovf_tok + base, sel, rhist, scan_scratch, binfo);
        for (int i = tid; i < kB; i += kFThreads) {
          const int ti = sel[i], c = ti / R, li = ti - c * R;
          dsm_red_or(dsm_addr(&umask[li >> 5], c), 1u << (li & 31));
        }
      }
    }
    cl.sync();  // D: the union bitmasks are complete
  } else if (k == T) {
    for (int w = tid; w < R / 32; w += kFThreads) {
      const int nb = min(32, max(0, n - 32 * w));
      umask[w] = nb == 32 ? 0xFFFFFFFFu : ((1u << nb) - 1u);
    }
    __syncthreads();
  } else {
    __syncthreads();
  }

  // ---- 4. output over this range
  // the union tokens of the range, ascending; their value refinement rows are
  // staged for the corrections
  if (warp == 0) {
    // warp 0 scans the bitmask: lane l holds words 2 l, 2 l + 1 (R <= 2048)
    const int nw = (n + 31) >> 5;
    uint32_t b0 = 2 * lane < nw ? umask[2 * lane] : 0u, b1 = 2 * lane + 1 < nw ? umask[2 * lane + 1] : 0u;
    const int cnt = __popc(b0) + __popc(b1);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = incl - cnt;
    while (b0) {
      const int b = __ffs(b0) - 1;
      b0 &= b0 - 1u;
      ulist[pos++] = static_cast<uint16_t>(64 * lane + b);
    }
    while (b1) {
      const int b = __ffs(b1) - 1;
      b1 &= b1 - 1u;
      ulist[pos++] = static_cast<uint16_t>(64 * lane + 32 + b);
    }
    if (lane == 31) ucnt = incl;
  }
  __syncthreads();
  const int nu = ucnt;
  for (int u = tid; u < min(nu, kFStgCap); u += kFThreads) {
    const uint32_t* src = a.v_ref + (row0 + ulist[u]) * kWordsPerRow;
    cp_async16_attn(stg + u * kWordsPerRow, src);
    cp_async16_attn(stg + u * kWordsPerRow + 4, src + 4);
  }
  cp_async_commit_attn();
  // refined scores of the union tokens from their full 4-bit key codes: four
  // lanes per token, lane q taking words q and q + 4 (32 dims) for every head
  // of the group (each code extracted once), summed over the four lanes
  cp_async_wait_attn<1>();  // the staged key rows (the value rows may still be in flight)
  __syncthreads();
  {
    const int qq = lane & 3;
    for (int base = 0; base < nu; base += kFThreads / 4) {  // uniform over the block: the shuffles
      const int u = base + (tid >> 2);
      const bool valid = u < nu;
      const int i = valid ? ulist[u] : 0;
      float P[GRP];
#pragma unroll
      for (int h = 0; h < GRP; ++h) P[h] = 0.0f;
      if (valid) {
        const int s = selecting ? smap[i] : 0xFF;
        const uint32_t* pr;
        const uint32_t* pf;
        if (s != 0xFF) {  // staged during the selection: resident words, then refinement words
          pr = kst + s * 2 * kWordsPerRow;
          pf = pr + kWordsPerRow;
        } else {
          pr = a.k_res + (row0 + i) * kWordsPerRow;
          pf = a.k_ref + (row0 + i) * kWordsPerRow;
        }
        const uint32_t r0 = pr[qq], r1 = pr[qq + 4], f0 = pf[qq], f1 = pf[qq + 4];
#pragma unroll
        for (int ww = 0; ww < 2; ++ww) {
          const int w = qq + 4 * ww;
          const uint32_t rw = ww ? r1 : r0, fw = ww ? f1 : f0;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float c = i2f_exact(static_cast<int>(((rw >> (2 * j)) & 3u) * 4u + ((fw >> (2 * j)) & 3u)));
#pragma unroll
            for (int h = 0; h < GRP; ++h) P[h] = fmaf(qs[h][16 * w + j], c, P[h]);
          }
        }
      }
#pragma unroll
      for (int h = 0; h < GRP; ++h) {
        P[h] += __shfl_xor_sync(0xffffffffu, P[h], 1);
        P[h] += __shfl_xor_sync(0xffffffffu, P[h], 2);
      }
      if (valid && qq == 0) {
        const uint32_t kz = ksz[i];
        const float sv = sfd::half_bits_to_float(static_cast<uint16_t>(kz & 0xFFFFu));
        const float z = sfd::half_bits_to_float(static_cast<uint16_t>(kz >> 16));
#pragma unroll
        for (int h = 0; h < GRP; ++h) sc[h * R + i] = (sv * fmaf(-z, qsm[h], P[h])) * kInvSqrtD;
      }
    }
  }
  __syncthreads();

  // the range's maximum score per head; the value stream starts meanwhile
  for (int i = 0; i < kFRing - 2; ++i) {
    if (tile0 + i < tile1) issue(a.v_res, tile0 + i);
    cp_async_commit_attn();
  }
  {
    float mx[GRP];
#pragma unroll
    for (int h = 0; h < GRP; ++h) mx[h] = -INFINITY;
    for (int i = tid; i < n; i += kFThreads)
#pragma unroll
      for (int h = 0; h < GRP; ++h) mx[h] = fmaxf(mx[h], sc[h * R + i]);
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const float m = warp_max(mx[h]);
      if (lane == 0) red[warp][h] = m;
    }
    __syncthreads();
    if (tid < GRP) {
      float m = -INFINITY;
#pragma unroll 1
      for (int w = 0; w < kFW; ++w) m = fmaxf(m, red[w][tid]);
      Msh[tid] = m;
    }
    __syncthreads();
  }

  // weights, in place over the scores: every score of this thread is read
  // before any weight is written
  float lsum[GRP], csum[GRP], asum[GRP];
#pragma unroll
  for (int h = 0; h < GRP; ++h) lsum[h] = csum[h] = asum[h] = 0.0f;
  {
    float M[GRP];
#pragma unroll
    for (int h = 0; h < GRP; ++h) M[h] = Msh[h];
    float pv[kPT][GRP];
#pragma unroll
    for (int j = 0; j < kPT; ++j) {
      const int i = tid + j * kFThreads;
#pragma unroll
      for (int h = 0; h < GRP; ++h) pv[j][h] = i < n ? sc[h * R + i] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kPT; ++j) {
      const int i = tid + j * kFThreads;
      if (i >= 16 * ntile) break;
      const bool valid = i < n;
      const uint32_t vz = valid ? vsz[i] : 0u;
      const float sv = sfd::half_bits_to_float(static_cast<uint16_t>(vz & 0xFFFFu));
      const float zv = sfd::half_bits_to_float(static_cast<uint16_t>(vz >> 16));
#pragma unroll
      for (int h = 0; h < GRP; ++h) {
        const float p = valid ? __expf(pv[j][h] - M[h]) : 0.0f;
        const float al = p * sv;
        const __half ahi = __float2half_rn(al);
        const __half alo = __float2half_rn(al - __half2float(ahi));
        as[h * kStr + i] = ahi;
        as[(GRP + h) * kStr + i] = alo;
        lsum[h] += p;
        csum[h] = fmaf(al, 1.5f - zv, csum[h]);
        asum[h] += __half2float(ahi) + __half2float(alo);
      }
#pragma unroll
      for (int h = 2 * GRP; h < NT * 8; ++h) as[h * kStr + i] = __float2half_rn(0.0f);
    }
    __syncthreads();
  }

  // value MMAs over this warp's tiles: o += (1024 + c) x alpha (f16 hi/lo columns)
  float acc[NT][8][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int w = 0; w < 8; ++w)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[nt][w][c] = 0.0f;
  for (int ti = tile0; ti < tile1; ti += 2) {
    if (ti + kFRing - 2 < tile1) issue(a.v_res, ti + kFRing - 2);
    cp_async_commit_attn();
    if (ti + kFRing - 1 < tile1) issue(a.v_res, ti + kFRing - 1);
    cp_async_commit_attn();
    cp_async_wait_attn<2>();
    __syncwarp();
    // a missing second tile reads a stale stage with zero weights: its
    // columns lie past this warp's tiles, so they are taken as zero here
    const bool two = ti + 1 < tile1;
    uint32_t b0[2][NT], b1[2][NT];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const __half* ar = as + (nt * 8 + g8) * kStr + 16 * (ti + u) + 2 * tig;
        b0[u][nt] = (u == 0 || two) ? *reinterpret_cast<const uint32_t*>(ar) : 0u;
        b1[u][nt] = (u == 0 || two) ? *reinterpret_cast<const uint32_t*>(ar + 8) : 0u;
      }
    // word g8 of token rows 2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9 of each
    // tile: MMA s covers dims 16 g8 + s and 16 g8 + 8 + s (vfrag)
    uint32_t src[2][4][4];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t* vr = ring + (warp * kFRing + (ti + u - tile0) % kFRing) * 16 * kWordsPerRow;
      vperm(vr[(2 * tig) * kWordsPerRow + g8], vr[(2 * tig + 1) * kWordsPerRow + g8],
            vr[(2 * tig + 8) * kWordsPerRow + g8], vr[(2 * tig + 9) * kWordsPerRow + g8], src[u]);
    }
#pragma unroll
    for (int s = 0; s < 8; ++s)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        uint32_t a0, a1, a2, a3;
        vfrag(src[u], s, a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_f16f32(acc[nt][s], a0, a1, a2, a3, b0[u][nt], b1[u][nt]);
      }
    __syncwarp();
  }
  cp_async_wait_attn<0>();
  __syncthreads();  // the staged refinement rows come from every thread

  // refined tokens: alpha (c_f - 1.5), lane = dims 4 lane .. 4 lane + 3
  float uo[GRP][4];
#pragma unroll
  for (int h = 0; h < GRP; ++h)
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) uo[h][dd] = 0.0f;
  for (int u = warp; u < nu; u += kFW) {
    const int i = ulist[u];
    const uint32_t wrow = u < kFStgCap ? stg[u * kWordsPerRow + (lane >> 2)]
                                       : a.v_ref[(row0 + i) * kWordsPerRow + (lane >> 2)];
    const uint32_t wf = wrow >> ((lane & 3) * 8);
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const float al = __half2float(as[h * kStr + i]) + __half2float(as[(GRP + h) * kStr + i]);
#pragma unroll
      for (int dd = 0; dd < 4; ++dd)
        uo[h][dd] = fmaf(al, i2f_exact(static_cast<int>((wf >> (2 * dd)) & 3u)) - 1.5f, uo[h][dd]);
    }
  }
  __syncthreads();  // every warp is done with the weight tile

  // this warp's output tile ww[head][dim] (in units of the code part, which
  // carries the factor 4^e of the dim's fragment position: uo enters as
  // uo 4^e / 2^b_f) in the dead weight tile; the high and low weight columns
  // of a head meet in one lane (or a lane pair)
  float* ww = reinterpret_cast<float*>(smem + S.sc) + warp * GRP * D;
#pragma unroll
  for (int w = 0; w < 8; ++w)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float v;
      bool st;
      int hh;
      if constexpr (GRP == 8) {
        v = acc[0][w][c] + acc[NT - 1][w][c];
        hh = 2 * tig + (c & 1);
        st = true;
      } else if constexpr (GRP == 1) {
        v = acc[0][w][c] + acc[0][w][c ^ 1];
        hh = 0;
        st = tig == 0 && (c & 1) == 0;
      } else {
        v = acc[0][w][c] + __shfl_xor_sync(0xffffffffu, acc[0][w][c], GRP / 2);
        hh = 2 * tig + (c & 1);
        st = tig < GRP / 2;
      }
      if (st) ww[hh * D + 16 * g8 + w + 8 * (c >> 1)] = v;  // MMA w, row g8 (+ 8)
    }
  __syncwarp();
#pragma unroll
  for (int h = 0; h < GRP; ++h)
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) ww[h * D + 4 * lane + dd] += (0.25f * vpos_mul(4 * lane + dd)) * uo[h][dd];
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    const float l = warp_sum(lsum[h]), cs = warp_sum(csum[h]), s = warp_sum(asum[h]);
    if (lane == 0) {
      red2[warp][h] = l;
      red2[warp][GRP + h] = cs;
      red2[warp][2 * GRP + h] = s;
    }
  }
  __syncthreads();
  float* gp = a.gpart + (static_cast<size_t>(g) * kFMaxCluster + r) * GRP * (D + 2);
  for (int e = tid; e < GRP * (D + 2); e += kFThreads) {
    const int h = e / (D + 2), j = e % (D + 2);
    float v;
    if (j == 0) {
      v = Msh[h];
    } else {
      float Lsum = 0.0f, Cs = 0.0f, A = 0.0f, o = 0.0f;
#pragma unroll 1
      for (int w = 0; w < kFW; ++w) {
        Lsum += red2[w][h];
        Cs += red2[w][GRP + h];
        A += red2[w][2 * GRP + h];
        if (j >= 2) o += reinterpret_cast<const float*>(smem + S.sc)[(w * GRP + h) * D + j - 2];
      }
      // resident value s (2^b_f c + m_f - z): code part 4 (acc - 1024 A) 4^-e,
      // offset part Cs
      const float f = j >= 2 ? vpos_inv(j - 2) : 1.0f;
      v = j == 1 ? Lsum : fmaf(4.0f * f, o, fmaf(-4096.0f * f, A, Cs));
    }
    gp[e] = v;
  }
  if (tid == 0) a.gcnt[g * kFMaxCluster + r] = nu;
  // E: every CTA's partials and union count are in the workspace (the cluster
  // barrier orders the global writes before the reads below); no shared
  // memory is read across CTAs after it, so CTAs leave independently
  cl.sync();

  // ---- merge over the cluster: CTA r writes its share of the group's outputs
  const float* gpg = a.gpart + static_cast<size_t>(g) * kFMaxCluster * GRP * (D + 2);
  if (warp == 0) {
    // union offset of this range and the group's union length
    const int cc = lane < C ? __ldcg(a.gcnt + g * kFMaxCluster + lane) : 0;
    int incl = cc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int U = __shfl_sync(0xffffffffu, incl, 31);
    if (lane == r) uoff = incl - cc;
    if (lane == 0 && r == 0) a.sel_n[g] = (selecting && flag_sh) ? -1 - U : U;
  } else if (warp == 1) {
    // the splits' rescale factors per head: lanes (head, CTA) in 16-lane halves
#pragma unroll 1
    for (int h0 = 0; h0 < GRP; h0 += 2) {
      const int h = h0 + (lane >> 4), c = lane & 15;
      const bool ok = h < GRP && c < C;
      const float m = ok ? __ldcg(gpg + (c * GRP + h) * (D + 2)) : -INFINITY;
      const float l = ok ? __ldcg(gpg + (c * GRP + h) * (D + 2) + 1) : 0.0f;
      float mx = m;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float f = m == -INFINITY ? 0.0f : __expf(m - mx);
      float ls = f * l;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
      if (ok) Fc[h][c] = f;
      if (h < GRP && c == 0) Lh[h] = ls;
    }
  }
  __syncthreads();
  {
    // outputs [r per, (r + 1) per) of the group, L threads per output, each
    // summing every L-th CTA's partial
    const int per = (GRP * D + C - 1) / C;
    int L = 1;
    while (L < kFMaxCluster && 2 * L * per <= kFThreads) L <<= 1;
    const int e1 = min(GRP * D, (r + 1) * per);
    for (int e0 = r * per; e0 < e1; e0 += kFThreads / L) {
      const int e = e0 + tid / L, part_i = tid % L;
      float A = 0.0f;
      int h = 0, d = 0;
      if (e < e1) {
        h = e / D;
        d = e % D;
#pragma unroll 4
        for (int c = part_i; c < C; c += L) A = fmaf(Fc[h][c], __ldcg(gpg + (c * GRP + h) * (D + 2) + 2 + d), A);
      }
      for (int o = L >> 1; o > 0; o >>= 1) A += __shfl_xor_sync(0xffffffffu, A, o);
      if (e < e1 && part_i == 0) a.out[(static_cast<size_t>(g) * GRP + h) * D + d] = A / Lh[h];
    }
  }
  {
    // the union holds at most k tokens per head (GRP k per group); the bound
    // guards the output row against corrupt scores
    int32_t* so = a.sel_out + static_cast<size_t>(g) * GRP * k;
    const int off = uoff, cap = GRP * k;
    for (int u = tid; u < nu && off + u < cap; u += kFThreads) so[off + u] = t0 + ulist[u];
  }
}

template <int GRP>
struct FusedPlan {
  int R = 0, C = 0;
  size_t smem = 0;
};

template <int GRP>
bool fused_plan(int T, FusedPlan<GRP>* p) {
  const int rmax = fused_rmax(GRP);
  int R = ((T + kFMaxCluster - 1) / kFMaxCluster + 31) / 32 * 32;
  if (R > rmax) return false;
  p->R = R;
  p->C = std::max(GRP, (T + R - 1) / R);
  p->smem = static_cast<size_t>(fused_smem(GRP, R).total);
  return p->C <= kFMaxCluster;
}

cudaLaunchConfig_t fused_config(dim3 grid, size_t smem, int C, cudaStream_t s, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// Whether clusters of this plan fit the device at all (cached per device and
// plan): the cluster needs C co-resident CTAs of this shared-memory size.
template <int GRP>
bool fused_fits(const FusedPlan<GRP>& p) {
  static std::mutex mu;
  static int cache_dev[64][kFMaxCluster + 1];  // 0 unknown, 1 yes, 2 no
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(mu);
  int& c = cache_dev[dev][p.C];
  if (c == 0) {
    cudaFuncSetAttribute(attn_fused_kernel<GRP>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaFuncSetAttribute(attn_fused_kernel<GRP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(fused_smem(GRP, fused_rmax(GRP)).total));
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = fused_config(dim3(p.C, 1), p.smem, p.C, nullptr, attr);
    int nclusters = 0;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&nclusters, attn_fused_kernel<GRP>, &cfg);
    c = (e == cudaSuccess && nclusters >= 1) ? 1 : 2;
    cudaGetLastError();  // a refused query leaves no sticky error
  }
  return c == 1;
}

template <int GRP>
sf_status fused_run(const uint16_t* q, int Hkv, int T, const sf_qkv* kv, int k, int32_t* sel_out,
                    int32_t* sel_n, float* out, double* ovf_key, int32_t* ovf_tok, int32_t* ovf_sel, float* gpart,
                    int32_t* gcnt, cudaStream_t s) {
  FusedPlan<GRP> p;
  if (!fused_plan<GRP>(T, &p) || !fused_fits<GRP>(p)) return SF_ENOTIMPL;
  FusedArgs a{};
  a.q = q;
  a.k_res = kv->k_res;
  a.k_ref = kv->k_ref;
  a.v_res = kv->v_res;
  a.v_ref = kv->v_ref;
  a.k_scale = kv->k_scale;
  a.k_zero = kv->k_zero;
  a.v_scale = kv->v_scale;
  a.v_zero = kv->v_zero;
  a.T = T;
  a.k = k;
  a.R = p.R;
  a.S = kv->row_stride > 0 ? kv->row_stride : T;
  a.sel_out = sel_out;
  a.sel_n = sel_n;
  a.out = out;
  a.ovf_key = ovf_key;
  a.ovf_tok = ovf_tok;
  a.ovf_sel = ovf_sel;
  a.gpart = gpart;
  a.gcnt = gcnt;
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = fused_config(dim3(p.C, Hkv), p.smem, p.C, s, attr);
  SF_CHECK_CUDA(cudaLaunchKernelEx(&cfg, attn_fused_kernel<GRP>, a));
  return sf::check_launch("attn_fused_kernel");
}

}  // namespace

namespace sf {

bool attn_fused_eligible(int Hq, int Hkv, int T) {
  if (Hkv < 1 || Hq % Hkv != 0) return false;
  switch (Hq / Hkv) {
    case 1: { FusedPlan<1> p; return fused_plan<1>(T, &p) && fused_fits<1>(p); }
    case 2: { FusedPlan<2> p; return fused_plan<2>(T, &p) && fused_fits<2>(p); }
    case 4: { FusedPlan<4> p; return fused_plan<4>(T, &p) && fused_fits<4>(p); }
    case 8: { FusedPlan<8> p; return fused_plan<8>(T, &p) && fused_fits<8>(p); }
    default: return false;
  }
}

sf_status attn_fused_run(const uint16_t* q, int Hq, int Hkv, int T, const sf_qkv* kv, int k, int32_t* sel_out,
                         int32_t* sel_n, float* out, double* ovf_key, int32_t* ovf_tok, int32_t* ovf_sel,
                         float* gpart, int32_t* gcnt, cudaStream_t s) {
  switch (Hq / Hkv) {
    case 1: return fused_run<1>(q, Hkv, T, kv, k, sel_out, sel_n, out, ovf_key, ovf_tok, ovf_sel, gpart, gcnt, s);
    case 2: return fused_run<2>(q, Hkv, T, kv, k, sel_out, sel_n, out, ovf_key, ovf_tok, ovf_sel, gpart, gcnt, s);
    case 4: return fused_run<4>(q, Hkv, T, kv, k, sel_out, sel_n, out, ovf_key, ovf_tok, ovf_sel, gpart, gcnt, s);
    case 8: return fused_run<8>(q, Hkv, T, kv, k, sel_out, sel_n, out, ovf_key, ovf_tok, ovf_sel, gpart, gcnt, s);
    default: return sf::fail(SF_ENOTIMPL, "attn_fused_run: Hq/Hkv must be 1, 2, 4 or 8");
  }
}

}  // namespace sf
