// allocate.cu -- Rate-Distortion Retention (SPHERICAL KV technical summary
// 2.2; arXiv abstract: keep/drop and precision tiers per token and head
// under a fixed budget, tier-homogeneous pages with lightweight metadata).
//
// Budget mode: every unprotected token offers three upgrade steps
// (drop->T2 180 B, T2->T1 16 B, T1->T0 316 B) with priority
// fp32((u * fp32(r^2)) * kappa_step).  All steps of a sequence are ordered by
// (priority desc, step asc, head asc, position asc) through a 64-bit
// composite key, and the longest prefix that fits the budget left after the
// protected tokens and a partial-page reserve is taken.  The cut is found by
// an exact weighted radix select (8 passes of 8 bits, byte-weighted
// histograms), so the result is the same as a full sort.
// Quota mode: per (seq, head), the same radix select finds the ranks q0,
// q0+q1, q0+q1+q2 of the (utility desc, position asc) order.
// Then: tiers, per-(unit, tier) counts, page plan (CSR offsets and per-tier
// free-list bases), row_of by a block scan, page ids and headers.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace skv {

typedef unsigned __int128 u128;

static inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t alloc_workspace_bytes(int B, int Hkv, long long Tmax) {
  const size_t U = (size_t)B * Hkv;
  const size_t nseg = U;
  size_t n = 0;
  n += al256(4 * U * (size_t)Tmax);
  n += al256(8 * nseg * 3 * 3);
  n += al256(8 * nseg * 3 * 256);
  n += al256(4 * U * 3);
  n += al256(4 * U * 3);
  n += al256(8 * (size_t)B);
  n += al256(U * (size_t)Tmax);
  n += al256(12 * U * (size_t)((Tmax + kRowChunk - 1) / kRowChunk));
  return n;
}

void alloc_carve(AllocParams& p, void* ws) {
  const size_t U = (size_t)p.B * p.Hkv;
  const size_t nseg = U;
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.keyw = reinterpret_cast<float*>(w);
  w += al256(4 * U * (size_t)p.Tmax);
  p.sel = reinterpret_cast<unsigned long long*>(w);
  w += al256(8 * nseg * 3 * 3);
  p.hist = reinterpret_cast<unsigned long long*>(w);
  w += al256(8 * nseg * 3 * 256);
  p.counts = reinterpret_cast<int32_t*>(w);
  w += al256(4 * U * 3);
  p.tbase = reinterpret_cast<int32_t*>(w);
  w += al256(4 * U * 3);
  p.pinned = reinterpret_cast<long long*>(w);
  w += al256(8 * (size_t)p.B);
  p.eff_protect = w;
  w += al256(U * (size_t)p.Tmax);
  p.ccounts = reinterpret_cast<int32_t*>(w);
}

// ---------------------------------------------------------------- keys --

// Outlier-aware protection: one warp per token; lane l holds dims 4l .. 4l+3
// (pairs 2l, 2l+1).  A key is an outlier when some pair has
// u = (rho / r) sqrt(d/2) > 4, twice the share grid's top level, tested
// exactly on the fp16 integers: (d/2) rho^2 > 16 R2.  The flag joins the
// caller's protection mask in eff_protect, which the key kernels then read.
__global__ void __launch_bounds__(256) outlier_protect_kernel(const __grid_constant__ AllocParams p) {
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= (long long)p.B * p.Hkv * p.Tmax) return;
  const long long t = w % p.Tmax;
  const int b = (int)(w / p.Tmax / p.Hkv);
  bool flag = false;
  if (t < p.seq_lens[b]) {  // uniform across the warp
    const uint2 kv = *reinterpret_cast<const uint2*>(p.K + w * kHeadDim + 4 * lane);
    const uint16_t k4[4] = {(uint16_t)(kv.x & 0xFFFF), (uint16_t)(kv.x >> 16),
                            (uint16_t)(kv.y & 0xFFFF), (uint16_t)(kv.y >> 16)};
    u128 a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const long long m = half_bits_to_m(k4[i]);
      a[i] = (u128)(m < 0 ? -m : m);
    }
    const u128 pr0 = a[0] * a[0] + a[1] * a[1], pr1 = a[2] * a[2] + a[3] * a[3];
    u128 sq = pr0 + pr1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long lo = (unsigned long long)sq, hi = (unsigned long long)(sq >> 64);
      const unsigned long long olo = __shfl_xor_sync(0xFFFFFFFFu, lo, o);
      const unsigned long long ohi = __shfl_xor_sync(0xFFFFFFFFu, hi, o);
      sq += ((u128)ohi << 64) | olo;
    }
    const u128 lim = (u128)16 * sq;
    constexpr unsigned kHalfD = kHeadDim / 2;
    flag = __any_sync(0xFFFFFFFFu, pr0 * kHalfD > lim || pr1 * kHalfD > lim);
  }
  if (lane == 0)
    p.eff_protect[w] = (uint8_t)(((p.protect != nullptr && p.protect[w] != 0) || flag) ? 1 : 0);
}

__device__ __forceinline__ float valid_utility(const AllocParams& p, long long i) {
  if (!p.utility) return 0.0f;
  float u = p.utility[i];
  if (!(u >= 0.0f) || isinf(u)) {
    report(p.err, SKV_ERR_ARG);
    return 0.0f;
  }
  return u;
}

// fp32(r^2) of a key from the warp's 32 lanes, each holding four of its fp16
// components (any assignment of components to lanes: the sum of squares is
// exact in 128-bit integers), rounded once to fp64 and once to fp32.
__device__ __forceinline__ float warp_r2f(uint2 kv) {
  const uint16_t k4[4] = {(uint16_t)(kv.x & 0xFFFF), (uint16_t)(kv.x >> 16),
                          (uint16_t)(kv.y & 0xFFFF), (uint16_t)(kv.y >> 16)};
  u128 sq = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long m = half_bits_to_m(k4[i]);
    const u128 a = (u128)(m < 0 ? -m : m);
    sq += a * a;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    unsigned long long lo = (unsigned long long)sq, hi = (unsigned long long)(sq >> 64);
    unsigned long long olo = __shfl_xor_sync(0xFFFFFFFFu, lo, o);
    unsigned long long ohi = __shfl_xor_sync(0xFFFFFFFFu, hi, o);
    sq += ((u128)ohi << 64) | olo;
  }
  const double r2 = u128_to_double_rn((unsigned long long)(sq >> 64), (unsigned long long)sq);
  return __double2float_rn(__dmul_rn(r2, 3.552713678800501e-15));  // 2^-48
}

// A token whose tier is fixed: keyw = -1 - tier (no upgrade steps), and its
// bytes count against the sequence's budget before the walk.
__device__ __forceinline__ void pin_token(const AllocParams& p, long long w, int b, int tier) {
  p.keyw[w] = -1.0f - (float)tier;
  if (tier < SKV_TIER_DROP)
    atomicAdd(reinterpret_cast<unsigned long long*>(&p.pinned[b]),
              (unsigned long long)tier_row_bytes(tier));
}

// budget mode: one warp per token; keyw = u * fp32(r^2), -1 when protected.
// Block x of a unit's nbx = ceil(Tmax / 8) blocks takes positions 8x .. 8x + 7
// (one 32-bit division per block, none per token).
__global__ void __launch_bounds__(256) keys_budget_kernel(const __grid_constant__ AllocParams p,
                                                          unsigned nbx) {
  const int lane = threadIdx.x & 31;
  const unsigned u = blockIdx.x / nbx;
  const long long t = (long long)(blockIdx.x - u * nbx) * 8 + (threadIdx.x >> 5);
  const int b = (int)(u / (unsigned)p.Hkv);
  if (t >= p.Tmax || t >= p.seq_lens[b]) return;
  const long long w = (long long)u * p.Tmax + t;
  if (p.protect && p.protect[w]) {
    if (lane == 0) pin_token(p, w, b, SKV_TIER_T0);
    return;
  }
  const float r2f = warp_r2f(*reinterpret_cast<const uint2*>(p.K + w * kHeadDim + 4 * lane));
  if (lane == 0) p.keyw[w] = __fmul_rn(valid_utility(p, w), r2f);
}

// re-tiering, one thread per (unit, position): a demoted token (T0 in the
// old store) gets the budget key from the fp16 key in its old T0 page (the
// row's component order does not matter for r^2: the sum is exact); every
// other resident token keeps its old tier (key -1 - tier) and its bytes are
// summed per block, one atomic per block (a block holds positions of one
// unit).  Demoted rows are few, so one thread computes a whole key's norm.
__global__ void __launch_bounds__(256) keys_retier_kernel(const __grid_constant__ AllocParams p,
                                                          unsigned nbx) {
  __shared__ unsigned long long sum;
  if (threadIdx.x == 0) sum = 0;
  __syncthreads();
  const unsigned u = blockIdx.x / nbx;
  const long long t = (long long)(blockIdx.x - u * nbx) * blockDim.x + threadIdx.x;
  const int b = (int)(u / (unsigned)p.Hkv);
  unsigned long long bytes = 0;
  if (t < p.Tmax && t < p.seq_lens[b]) {
    const long long w = (long long)u * p.Tmax + t;
    const int to = p.tier_old[w];
    if (to > SKV_TIER_DROP) {
      report(p.err, SKV_ERR_CORRUPT);
      p.keyw[w] = -1.0f - (float)SKV_TIER_DROP;
    } else if (!p.demote[w] || to != SKV_TIER_T0) {
      if (p.demote[w]) report(p.err, SKV_ERR_ARG);  // only T0 rows can be demoted
      p.keyw[w] = -1.0f - (float)to;
      bytes = to < SKV_TIER_DROP ? (unsigned long long)tier_row_bytes(to) : 0ull;
    } else {
      const int row = p.row_old[w];
      const long long gi = (long long)p.indptr_old[u] + (row >= 0 ? row / p.P : 0);
      const uint32_t id = row >= 0 && gi < p.tindptr_old[3 * u + 1] && gi < p.page_cap
                              ? p.ids_old[gi] : 0xFFFFFFFFu;
      const uint32_t slot = id & 0x3FFFFFFFu;
      if ((id >> 30) != 0u || (long long)slot >= p.slots[0]) {
        report(p.err, SKV_ERR_CORRUPT);
        p.keyw[w] = -1.0f - (float)SKV_TIER_DROP;
      } else {
        const uint4* krow = reinterpret_cast<const uint4*>(
            p.pool[0] + (long long)slot * p.stride[0] + kHdrBytes + 256 * (row % p.P));
        u128 sq = 0;
        for (int c = 0; c < 16; ++c) {
          const uint4 v = krow[c];
          const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const long long m = half_bits_to_m((wd[k >> 1] >> (16 * (k & 1))) & 0xFFFFu);
            const u128 a = (u128)(m < 0 ? -m : m);
            sq += a * a;
          }
        }
        const double r2 = u128_to_double_rn((unsigned long long)(sq >> 64), (unsigned long long)sq);
        const float r2f = __double2float_rn(__dmul_rn(r2, 3.552713678800501e-15));  // 2^-48
        p.keyw[w] = __fmul_rn(valid_utility(p, w), r2f);
      }
    }
  }
  if (bytes) atomicAdd(&sum, bytes);
  __syncthreads();
  if (threadIdx.x == 0 && sum)
    atomicAdd(reinterpret_cast<unsigned long long*>(&p.pinned[b]), sum);
}

// quota mode: keyw = u (0 without utilities), -1 when protected
__global__ void keys_quota_kernel(const __grid_constant__ AllocParams p) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)p.B * p.Hkv * p.Tmax) return;
  const long long t = i % p.Tmax;
  const int b = (int)(i / p.Tmax / p.Hkv);
  if (t >= p.seq_lens[b]) return;
  p.keyw[i] = (p.protect && p.protect[i]) ? -1.0f : valid_utility(p, i);
}

// ---------------------------------------------------------- radix select --

// state per (segment, target): [0] prefix, [1] remaining (int64 bits), [2] done
__global__ void sel_init_kernel(const __grid_constant__ AllocParams p) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= p.nseg * 3) return;
  const int seg = i / 3, j = i % 3;
  unsigned long long* st = p.sel + (size_t)i * 3;
  st[0] = 0;
  st[1] = 0;
  st[2] = 0;
  if (p.mode == SKV_MODE_BUDGET) {
    if (j != 0) {
      st[2] = 1;
      return;
    }
    const long long reserve = (long long)p.Hkv * (p.P - 1) * (512 + 196 + 180);
    const long long left = p.budget[seg] - p.pinned[seg] - reserve;
    if (left < 0) {
      report(p.err, SKV_ERR_BUDGET);
      st[2] = 1;  // prefix 0: nothing is selected
      return;
    }
    st[1] = (unsigned long long)left;
  } else {
    const int b = seg / p.Hkv;
    const long long q0 = p.quota[3 * b], q1 = p.quota[3 * b + 1], q2 = p.quota[3 * b + 2];
    if (q0 < 0 || q1 < 0 || q2 < 0) {
      report(p.err, SKV_ERR_ARG);
      st[2] = 1;
      return;
    }
    st[1] = (unsigned long long)(j == 0 ? q0 : (j == 1 ? q0 + q1 : q0 + q1 + q2));
  }
}

// 64-bit composite of budget step k of token (h, t) with weight w: the
// priority fp32(w kappa_k) descending, then step, head, position ascending
__device__ __forceinline__ unsigned long long budget_comp(const AllocParams& p, float w, int k,
                                                         int h, long long t) {
  const float key = __fmul_rn(w, p.kappa[k]);
  return ((unsigned long long)(0xFFFFFFFFu - __float_as_uint(key)) << 32) |
         ((unsigned long long)k << 30) | ((unsigned long long)h << 23) | (unsigned long long)t;
}

constexpr int kHistItemsPerBlock = 4096;  // tokens (budget) or positions (quota) per block

// Weighted histogram of one 8-bit digit of the composites that still match
// each target's prefix.  Budget mode: a thread per token (h, t) of sequence
// seg with its three steps (weights 180, 16, 316 bytes); quota mode: a thread
// per position of unit seg (weight 1, three targets).  Every lane of a warp
// runs the same number of rounds (the tail lanes with nothing), so the lanes
// that add to the same bin are grouped: one shared atomic per group and
// round instead of one per lane (the early passes put nearly every item into
// a few bins).
__global__ void __launch_bounds__(256) hist_kernel(const __grid_constant__ AllocParams p,
                                                   int shift) {
  __shared__ unsigned long long sh[3][256];
  __shared__ unsigned long long pre[3];
  __shared__ int dn[3];
  const int seg = blockIdx.y;
  const bool budget = p.mode == SKV_MODE_BUDGET;
  const int ntgt = budget ? 1 : 3;
  if (threadIdx.x < 3) {
    const unsigned long long* st = p.sel + ((size_t)seg * 3 + threadIdx.x) * 3;
    pre[threadIdx.x] = st[0];
    dn[threadIdx.x] = (threadIdx.x < ntgt) ? (int)st[2] : 1;
  }
  for (int i = threadIdx.x; i < 3 * 256; i += blockDim.x) (&sh[0][0])[i] = 0;
  __syncthreads();
  if (dn[0] && dn[1] && dn[2]) return;
  const long long n = budget ? (long long)p.Hkv * p.Tmax : p.Tmax;
  const long long i0 = (long long)blockIdx.x * kHistItemsPerBlock;
  const long long i1 = min(n, i0 + kHistItemsPerBlock);
  const int lane = threadIdx.x & 31;
  for (long long base = i0; base < i1; base += blockDim.x) {
    const long long i = base + threadIdx.x;
    if (budget) {
      // token i = h Tmax + t of sequence seg (Hkv Tmax < 2^31: 32-bit division)
      int h = 0;
      long long t = 0;
      float w = -1.0f;
      if (i < i1) {
        h = (int)((unsigned)i / (unsigned)p.Tmax);
        t = i - (long long)h * p.Tmax;
        if (t < p.seq_lens[seg]) w = p.keyw[(long long)seg * n + i];
      }
      const bool have = w >= 0.0f && !dn[0];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const unsigned long long comp = have ? budget_comp(p, w, k, h, t) : 0ull;
        const int dig = (int)((comp >> shift) & 255u);
        const bool in = have && (shift >= 56 || (comp >> (shift + 8)) == (pre[0] >> (shift + 8)));
        const uint32_t peers = __match_any_sync(0xFFFFFFFFu, in ? (uint32_t)dig : ~0u);
        if (in && lane == __ffs(peers) - 1)
          atomicAdd(&sh[0][dig], (unsigned long long)(k == 0 ? 180u : (k == 1 ? 16u : 316u)) *
                                     (unsigned long long)__popc(peers));
      }
    } else {
      const int b = seg / p.Hkv;
      float w = -1.0f;
      if (i < i1 && i < p.seq_lens[b]) w = p.keyw[(long long)seg * p.Tmax + i];
      const unsigned long long comp =
          ((unsigned long long)(0xFFFFFFFFu - __float_as_uint(w)) << 32) | (unsigned long long)i;
      const int dig = (int)((comp >> shift) & 255u);
      for (int j = 0; j < 3; ++j) {
        const bool in = w >= 0.0f && !dn[j] &&
                        (shift >= 56 || (comp >> (shift + 8)) == (pre[j] >> (shift + 8)));
        const uint32_t peers = __match_any_sync(0xFFFFFFFFu, in ? (uint32_t)dig : ~0u);
        if (in && lane == __ffs(peers) - 1)
          atomicAdd(&sh[j][dig], (unsigned long long)__popc(peers));
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < ntgt * 256; i += blockDim.x) {
    const unsigned long long v = (&sh[0][0])[i];
    if (v) atomicAdd(&p.hist[(size_t)seg * 3 * 256 + i], v);
  }
}

// One block of 256 threads per (segment, target): bin d of the histogram is
// thread d's; a block-wide inclusive scan finds the one digit at which the
// target's remaining weight falls (the cumulative weight before it at most
// the remainder, with it above), and every bin is cleared for the next pass.
__global__ void __launch_bounds__(256) sel_step_kernel(const __grid_constant__ AllocParams p,
                                                       int shift) {
  __shared__ unsigned long long wsum[8];
  const int i = blockIdx.x;
  if (i >= p.nseg * 3) return;  // uniform over the block
  const int d = threadIdx.x, lane = d & 31, wid = d >> 5;
  unsigned long long* st = p.sel + (size_t)i * 3;
  unsigned long long* h = p.hist + (size_t)i * 256;
  const unsigned long long v = h[d];
  h[d] = 0;
  const bool done = st[2] != 0;
  const unsigned long long rem = st[1];
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[wid] = x;
  __syncthreads();  // every thread has read st before any writes it
  unsigned long long before = 0;
  for (int k = 0; k < wid; ++k) before += wsum[k];
  const unsigned long long incl = before + x, excl = incl - v;
  if (done) return;
  if (excl <= rem && incl > rem) {  // at most one thread
    st[0] |= (unsigned long long)d << shift;
    st[1] = rem - excl;
  }
  if (d == 255 && incl <= rem) {
    st[2] = 1;
    st[0] = ~0ull;  // every item is below the cut
  }
}

// ------------------------------------------------------------------ tiers --

__global__ void tier_kernel(const __grid_constant__ AllocParams p) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)p.B * p.Hkv * p.Tmax) return;
  const long long t = i % p.Tmax;
  const long long bh = i / p.Tmax;
  const int h = (int)(bh % p.Hkv), b = (int)(bh / p.Hkv);
  uint8_t tr = SKV_TIER_DROP;
  if (t < p.seq_lens[b]) {
    const float w = p.keyw[i];
    if (w < 0.0f) {
      tr = (uint8_t)(-1 - (int)w);  // a fixed tier
    } else if (p.mode == SKV_MODE_BUDGET) {
      const unsigned long long cut = p.sel[(size_t)b * 3 * 3 + 0];
      int lvl = 0;
#pragma unroll
      for (int k = 0; k < 3; ++k) lvl += budget_comp(p, w, k, h, t) < cut;
      tr = lvl == 3 ? SKV_TIER_T0 : (lvl == 2 ? SKV_TIER_T1 : (lvl == 1 ? SKV_TIER_T2 : SKV_TIER_DROP));
    } else {
      const unsigned long long comp =
          ((unsigned long long)(0xFFFFFFFFu - __float_as_uint(w)) << 32) | (unsigned long long)t;
      const unsigned long long* st = p.sel + (size_t)bh * 3 * 3;
      if (comp < st[0]) tr = SKV_TIER_T0;
      else if (comp < st[3]) tr = SKV_TIER_T1;
      else if (comp < st[6]) tr = SKV_TIER_T2;
    }
  }
  p.tier_out[i] = tr;
  if (tr == SKV_TIER_DROP) p.row_of[i] = -1;
}

// -------------------------------------------------------- counts and plan --

// Tier counts per (unit, chunk of kRowChunk positions) into ccounts, and per
// unit (counts, zeroed before) by atomics.  Grid: x the chunks, y a stride
// over the units.
__global__ void __launch_bounds__(256) unit_count_kernel(const __grid_constant__ AllocParams p) {
  __shared__ int c[3];
  const int U = p.B * p.Hkv;
  const int nch = (int)((p.Tmax + kRowChunk - 1) / kRowChunk);
  const long long t0 = (long long)blockIdx.x * kRowChunk;
  for (int u = blockIdx.y; u < U; u += gridDim.y) {
    if (threadIdx.x < 3) c[threadIdx.x] = 0;
    __syncthreads();
    const long long T = p.seq_lens[u / p.Hkv];
    const long long t1 = min(T, t0 + kRowChunk);
    int l0 = 0, l1 = 0, l2 = 0;
    for (long long t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
      if (p.dense) {
        ++l0;
        continue;
      }
      const uint8_t tr = p.tier_out[(long long)u * p.Tmax + t];
      l0 += tr == 0;
      l1 += tr == 1;
      l2 += tr == 2;
    }
    if (l0) atomicAdd(&c[0], l0);
    if (l1) atomicAdd(&c[1], l1);
    if (l2) atomicAdd(&c[2], l2);
    __syncthreads();
    if (threadIdx.x < 3) {
      const int v = c[threadIdx.x];
      p.ccounts[((long long)u * nch + blockIdx.x) * 3 + threadIdx.x] = v;
      if (v) atomicAdd(&p.counts[u * 3 + threadIdx.x], v);
    }
    __syncthreads();
  }
}

// block-wide exclusive scan of long long (blockDim.x = 1024)
__device__ long long block_exclusive_scan(long long v, long long& total) {
  __shared__ long long wsum[32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[wid] = x;
  __syncthreads();
  if (wid == 0) {
    const int nw = blockDim.x >> 5;
    long long s = lane < nw ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xFFFFFFFFu, s, o);
      if (lane >= o) s += y;
    }
    wsum[lane] = s;
  }
  __syncthreads();
  const long long before = (wid > 0 ? wsum[wid - 1] : 0) + x - v;
  total = wsum[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before;
}

// re-tiering: the first row of each (unit, tier) segment at which the new
// store differs from the old one -- a new row holding another token than
// the old row of that index, or an old row whose token moved or left (rows
// counted within the segment).  Rows of a segment are in position order in
// both stores, so every page wholly before that row is byte-identical in
// both (rows, count and header) and stays where it is.
__global__ void diff_kernel(const __grid_constant__ AllocParams p) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)p.B * p.Hkv * p.Tmax) return;
  const long long t = i % p.Tmax, u = i / p.Tmax;
  if (t >= p.seq_lens[u / p.Hkv]) return;
  const int tn = p.tier_out[i], to = p.tier_old[i];
  // row within the tier's segment: row_of counts from the unit's first page,
  // so the segment's page base (the pages of the tiers before it) comes off
  const int P = p.P;
  int rn = -1, ro = -1;
  if (tn < SKV_TIER_DROP) {
    const int c0 = p.counts[3 * u], c1 = p.counts[3 * u + 1];
    const int pb = tn == 0 ? 0 : (c0 + P - 1) / P + (tn == 2 ? (c1 + P - 1) / P : 0);
    rn = p.row_of[i] - pb * P;
  }
  if (to < SKV_TIER_DROP)
    ro = p.row_old[i] - (p.tindptr_old[3 * u + to] - p.indptr_old[u]) * P;
  if (tn == to && rn == ro) return;
  if (tn < SKV_TIER_DROP) atomicMin(&p.diff[3 * u + tn], max(rn, 0));
  if (to < SKV_TIER_DROP) atomicMin(&p.diff[3 * u + to], max(ro, 0));
}

// CSR offsets of the new page table and, per (unit, tier), the first index
// into the tier's free list.  A re-tiering keeps each segment's leading
// unchanged pages (keep), takes free slots only for the others (from the
// list's cursor on) and lists the old pages it no longer references.
__global__ void __launch_bounds__(1024) page_plan_kernel(const __grid_constant__ AllocParams p) {
  const int U = p.B * p.Hkv;
  const int per = (U + blockDim.x - 1) / blockDim.x;
  const int u0 = threadIdx.x * per, u1 = min(U, u0 + per);
  const bool rt = p.keep != nullptr;
  long long cur[3] = {0, 0, 0};
  if (rt)
    for (int t = 0; t < 3; ++t) cur[t] = p.cursor[t];
  // s[0..2]: free slots taken per tier, s[3]: pages, s[4]: old pages released
  long long s[5] = {0, 0, 0, 0, 0};
  for (int u = u0; u < u1; ++u) {
    for (int t = 0; t < 3; ++t) {
      const long long np = (p.counts[u * 3 + t] + p.P - 1) / p.P;
      long long kp = 0;
      if (rt) {
        const long long npo = p.tindptr_old[3 * u + t + 1] - p.tindptr_old[3 * u + t];
        kp = min(min((long long)p.diff[3 * u + t] / p.P, np), npo);
        p.keep[3 * u + t] = (int32_t)kp;
        s[4] += npo - kp;
      }
      s[t] += np - kp;
      s[3] += np;
    }
  }
  long long base[5], tot[5];
  for (int k = 0; k < 5; ++k) base[k] = block_exclusive_scan(s[k], tot[k]);
  for (int u = u0; u < u1; ++u) {
    p.indptr[u] = (int32_t)base[3];
    if (rt) p.rbase[u] = (int32_t)base[4];
    for (int t = 0; t < 3; ++t) {
      if (p.tier_indptr) p.tier_indptr[u * 3 + t] = (int32_t)base[3];
      p.tbase[u * 3 + t] = (int32_t)(cur[t] + base[t]);
      const long long np = (p.counts[u * 3 + t] + p.P - 1) / p.P;
      base[t] += np - (rt ? p.keep[3 * u + t] : 0);
      base[3] += np;
    }
  }
  if (threadIdx.x == 0) {
    p.indptr[U] = (int32_t)tot[3];
    if (p.tier_indptr) p.tier_indptr[3 * U] = (int32_t)tot[3];
    bool bad = tot[3] > p.page_cap || tot[3] > 0x7FFFFFFFLL;
    for (int t = 0; t < 3; ++t) bad |= cur[t] < 0 || cur[t] + tot[t] > p.free_len[t];
    if (bad) report(p.err, SKV_ERR_POOL);
    if (rt) {
      for (int t = 0; t < 3; ++t) p.cursor[t] = (int32_t)(cur[t] + tot[t]);
      *p.n_released = (int32_t)tot[4];
    }
  }
}

// Row map, one block per (unit, chunk of kRowChunk positions): the chunk's
// rank base per tier is the sum of the unit's earlier chunks' counts, and a
// block scan ranks its positions (three 21-bit fields: a chunk holds at most
// 1024 of each tier).
__global__ void __launch_bounds__(1024) row_of_kernel(const __grid_constant__ AllocParams p) {
  const int U = p.B * p.Hkv;
  const int nch = (int)((p.Tmax + kRowChunk - 1) / kRowChunk);
  const int ch = blockIdx.x;
  const int P = p.P;
  for (int u = blockIdx.y; u < U; u += gridDim.y) {
    const long long T = p.seq_lens[u / p.Hkv];
    if ((long long)ch * kRowChunk >= T) continue;  // uniform over the block
    long long s0 = 0, s1 = 0, s2 = 0;
    for (int c = threadIdx.x; c < ch; c += blockDim.x) {
      const int32_t* cc = p.ccounts + ((long long)u * nch + c) * 3;
      s0 += cc[0];
      s1 += cc[1];
      s2 += cc[2];
    }
    long long base[3];
    block_exclusive_scan(s0, base[0]);
    block_exclusive_scan(s1, base[1]);
    block_exclusive_scan(s2, base[2]);
    const long long c0 = p.counts[u * 3], c1 = p.counts[u * 3 + 1];
    const long long pb[3] = {0, (c0 + P - 1) / P, (c0 + P - 1) / P + (c1 + P - 1) / P};
    const long long t = (long long)ch * kRowChunk + threadIdx.x;
    const long long i = (long long)u * p.Tmax + t;
    int tr = SKV_TIER_DROP;
    if (t < T) tr = p.tier_out[i];
    const long long f = tr == 0 ? 1LL : (tr == 1 ? (1LL << 21) : (tr == 2 ? (1LL << 42) : 0LL));
    long long tot;
    const long long ex = block_exclusive_scan(f, tot);
    if (t < T && tr < 3) {
      const long long rank = base[tr] + ((ex >> (21 * tr)) & ((1LL << 21) - 1));
      p.row_of[i] = (int32_t)((pb[tr] + rank / P) * P + rank % P);
    }
  }
}

// one warp per page: page id, header, zeroed payload for a partial page
__global__ void __launch_bounds__(256) page_write_kernel(const __grid_constant__ AllocParams p) {
  const int U = p.B * p.Hkv;
  const long long total = p.indptr[U];
  const int lane = threadIdx.x & 31;
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long g = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; g < total;
       g += nwarps) {
    int lo = 0, hi = U;  // largest u with indptr[u] <= g
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.indptr[mid] <= g) lo = mid; else hi = mid;
    }
    const int u = lo;
    const int P = p.P;
    const long long local = g - p.indptr[u];
    const long long n0 = p.counts[u * 3], n1 = p.counts[u * 3 + 1], n2 = p.counts[u * 3 + 2];
    const long long np0 = (n0 + P - 1) / P, np1 = (n1 + P - 1) / P;
    int t;
    long long pg, n;
    if (local < np0) { t = 0; pg = local; n = n0; }
    else if (local < np0 + np1) { t = 1; pg = local - np0; n = n1; }
    else { t = 2; pg = local - np0 - np1; n = n2; }
    const long long kp = p.keep ? p.keep[u * 3 + t] : 0;
    if (pg < kp) {  // an unchanged page of a re-tiered store: it stays
      const long long go = p.tindptr_old[3 * u + t] + pg;
      if (lane == 0) {
        if (g < p.page_cap && go >= 0 && go < p.page_cap) p.page_ids[g] = p.ids_old[go];
        else report(p.err, SKV_ERR_CORRUPT);
      }
      continue;
    }
    const long long fi = p.tbase[u * 3 + t] + pg - kp;
    if (g >= p.page_cap || fi >= p.free_len[t]) {
      if (lane == 0) report(p.err, SKV_ERR_POOL);
      continue;
    }
    const uint32_t slot = p.free_ids[t][fi];
    if ((long long)slot >= p.slots[t] || slot > 0x3FFFFFFFu) {
      if (lane == 0) report(p.err, SKV_ERR_POOL);
      continue;
    }
    if (lane == 0) p.page_ids[g] = ((uint32_t)t << 30) | slot;
    const int cnt = (int)min((long long)P, n - pg * P);
    uint8_t* page = p.pool[t] + (long long)slot * p.stride[t];
    if (cnt < P) {
      for (int o = kHdrBytes + 16 * lane; o < p.payload[t]; o += 32 * 16)
        *reinterpret_cast<uint4*>(page + o) = make_uint4(0, 0, 0, 0);
    }
    if (lane == 0) {
      uint4 hdr;
      hdr.x = (uint32_t)cnt | ((uint32_t)t << 16) | ((uint32_t)kPageMagic << 24);
      hdr.y = (uint32_t)(u / p.Hkv);
      hdr.z = (uint32_t)(u % p.Hkv);
      hdr.w = (uint32_t)pg;
      *reinterpret_cast<uint4*>(page) = hdr;
    }
  }
}

// re-tiering: the ids of the old pages that the new store no longer holds,
// per unit in (tier, page) order from rbase[u] on
__global__ void release_kernel(const __grid_constant__ AllocParams p) {
  const int U = p.B * p.Hkv;
  const long long n_old = min((long long)p.indptr_old[U], p.page_cap);
  const long long nthr = (long long)gridDim.x * blockDim.x;
  for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < n_old; g += nthr) {
    int lo = 0, hi = U - 1;  // the unit u with indptr_old[u] <= g < indptr_old[u + 1]
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.indptr_old[mid] <= g) lo = mid; else hi = mid - 1;
    }
    const int u = lo;
    long long idx = p.rbase[u];
    for (int t = 0; t < 3; ++t) {
      const long long a = p.tindptr_old[3 * u + t], e = p.tindptr_old[3 * u + t + 1];
      const long long kp = p.keep[3 * u + t];
      if (g < e) {
        const long long r = idx + (g - a - kp);
        if (g - a >= kp && r >= 0 && r < p.page_cap) p.released[r] = p.ids_old[g];
        break;
      }
      idx += (e - a) - kp;
    }
  }
}

static unsigned grid_for(long long n, int threads) {
  long long b = (n + threads - 1) / threads;
  return (unsigned)(b < 1 ? 1 : b);
}

// chunks of positions (x) by a stride over the units (y)
static dim3 row_grid(const AllocParams& p) {
  const long long nch = (p.Tmax + kRowChunk - 1) / kRowChunk;
  const long long U = (long long)p.B * p.Hkv;
  return dim3((unsigned)(nch < 1 ? 1 : nch), (unsigned)std::max(1LL, std::min(U, 65535LL)));
}

static cudaError_t launch_counts(AllocParams& p, cudaStream_t stream) {
  const size_t U = (size_t)p.B * p.Hkv;
  cudaError_t e = cudaMemsetAsync(p.counts, 0, 4 * 3 * U, stream);
  if (e != cudaSuccess) return e;
  if (U > 0) unit_count_kernel<<<row_grid(p), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_allocate(AllocParams& p, cudaStream_t stream) {
  const long long ntok = (long long)p.B * p.Hkv * p.Tmax;
  const int U = p.B * p.Hkv;
  p.dense = 0;
  p.nseg = p.mode == SKV_MODE_BUDGET ? p.B : U;
  cudaError_t e;
  if ((e = cudaMemsetAsync(p.pinned, 0, 8 * (size_t)p.B, stream)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.hist, 0, 8 * (size_t)p.nseg * 3 * 256, stream)) != cudaSuccess)
    return e;
  if (p.outlier && ntok > 0) {
    outlier_protect_kernel<<<grid_for(ntok * 32, 256), 256, 0, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    p.protect = p.eff_protect;  // the key kernels read the joined mask
  }
  if (ntok > 0) {
    if (p.mode == SKV_MODE_BUDGET) {
      const long long nbx = (p.Tmax + 7) / 8;
      if ((long long)U * nbx > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
      keys_budget_kernel<<<(unsigned)(U * nbx), 256, 0, stream>>>(p, (unsigned)nbx);
    }
    else
      keys_quota_kernel<<<grid_for(ntok, 256), 256, 0, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  sel_init_kernel<<<grid_for(p.nseg * 3, 128), 128, 0, stream>>>(p);
  const long long n_items = p.mode == SKV_MODE_BUDGET ? (long long)p.Hkv * p.Tmax : p.Tmax;
  const dim3 hgrid(grid_for(n_items, kHistItemsPerBlock), p.nseg);
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    hist_kernel<<<hgrid, 256, 0, stream>>>(p, shift);
    sel_step_kernel<<<std::max(1, p.nseg * 3), 256, 0, stream>>>(p, shift);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (ntok > 0) tier_kernel<<<grid_for(ntok, 256), 256, 0, stream>>>(p);
  if ((e = launch_counts(p, stream)) != cudaSuccess) return e;
  page_plan_kernel<<<1, 1024, 0, stream>>>(p);
  row_of_kernel<<<row_grid(p), 1024, 0, stream>>>(p);
  page_write_kernel<<<grid_for(std::min<long long>(p.page_cap, 1LL << 22) * 32, 256), 256, 0,
                      stream>>>(p);
  return cudaGetLastError();
}

size_t retier_workspace_bytes(int B, int Hkv, long long Tmax, long long page_cap) {
  const size_t U = (size_t)B * Hkv;
  return alloc_workspace_bytes(B, Hkv, Tmax) + al256(U * (size_t)Tmax) +
         al256(4 * U * (size_t)Tmax) + al256(4 * (U + 1)) + al256(4 * (3 * U + 1)) +
         al256(4 * (size_t)page_cap) + 2 * al256(4 * 3 * U) + al256(4 * U);
}

void retier_carve(AllocParams& p, void* ws) {
  const size_t U = (size_t)p.B * p.Hkv;
  alloc_carve(p, ws);
  uint8_t* w = static_cast<uint8_t*>(ws) + alloc_workspace_bytes(p.B, p.Hkv, p.Tmax);
  p.tier_old = w;
  w += al256(U * (size_t)p.Tmax);
  p.row_old = reinterpret_cast<int32_t*>(w);
  w += al256(4 * U * (size_t)p.Tmax);
  p.indptr_old = reinterpret_cast<int32_t*>(w);
  w += al256(4 * (U + 1));
  p.tindptr_old = reinterpret_cast<int32_t*>(w);
  w += al256(4 * (3 * U + 1));
  p.ids_old = reinterpret_cast<uint32_t*>(w);
  w += al256(4 * (size_t)p.page_cap);
  p.diff = reinterpret_cast<int32_t*>(w);
  w += al256(4 * 3 * U);
  p.keep = reinterpret_cast<int32_t*>(w);
  w += al256(4 * 3 * U);
  p.rbase = reinterpret_cast<int32_t*>(w);
}

cudaError_t launch_retier_plan(AllocParams& p, cudaStream_t stream) {
  const long long ntok = (long long)p.B * p.Hkv * p.Tmax;
  const int U = p.B * p.Hkv;
  p.dense = 0;
  p.mode = SKV_MODE_BUDGET;
  p.nseg = p.B;
  cudaError_t e;
  // the store as it is: every later step reads the old layout from here
  const size_t tok = (size_t)ntok;
  if ((e = cudaMemcpyAsync(p.tier_old, p.tier_out, tok, cudaMemcpyDeviceToDevice, stream)) ||
      (e = cudaMemcpyAsync(p.row_old, p.row_of, 4 * tok, cudaMemcpyDeviceToDevice, stream)) ||
      (e = cudaMemcpyAsync(p.indptr_old, p.indptr, 4 * ((size_t)U + 1), cudaMemcpyDeviceToDevice,
                           stream)) ||
      (e = cudaMemcpyAsync(p.tindptr_old, p.tier_indptr, 4 * (3 * (size_t)U + 1),
                           cudaMemcpyDeviceToDevice, stream)) ||
      (e = cudaMemcpyAsync(p.ids_old, p.page_ids, 4 * (size_t)p.page_cap,
                           cudaMemcpyDeviceToDevice, stream)))
    return e;
  if ((e = cudaMemsetAsync(p.pinned, 0, 8 * (size_t)p.B, stream)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.hist, 0, 8 * (size_t)p.nseg * 3 * 256, stream)) != cudaSuccess)
    return e;
  if ((e = cudaMemsetAsync(p.diff, 0x7F, 4 * 3 * (size_t)U, stream)) != cudaSuccess) return e;
  if (ntok > 0) {
    const long long nbx = (p.Tmax + 255) / 256;
    if ((long long)U * nbx > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    keys_retier_kernel<<<(unsigned)(U * nbx), 256, 0, stream>>>(p, (unsigned)nbx);
  }
  sel_init_kernel<<<grid_for(p.nseg * 3, 128), 128, 0, stream>>>(p);
  const dim3 hgrid(grid_for((long long)p.Hkv * p.Tmax, kHistItemsPerBlock), p.nseg);
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    hist_kernel<<<hgrid, 256, 0, stream>>>(p, shift);
    sel_step_kernel<<<std::max(1, p.nseg * 3), 256, 0, stream>>>(p, shift);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (ntok > 0) tier_kernel<<<grid_for(ntok, 256), 256, 0, stream>>>(p);
  if ((e = launch_counts(p, stream)) != cudaSuccess) return e;
  row_of_kernel<<<row_grid(p), 1024, 0, stream>>>(p);
  if (ntok > 0) diff_kernel<<<grid_for(ntok, 256), 256, 0, stream>>>(p);
  page_plan_kernel<<<1, 1024, 0, stream>>>(p);
  page_write_kernel<<<grid_for(std::min<long long>(p.page_cap, 1LL << 22) * 32, 256), 256, 0,
                      stream>>>(p);
  release_kernel<<<grid_for(std::min<long long>(p.page_cap, 1LL << 20), 256), 256, 0, stream>>>(
      p);
  return cudaGetLastError();
}

cudaError_t launch_dense_plan(AllocParams& p, cudaStream_t stream) {
  p.dense = 1;
  cudaError_t e = launch_counts(p, stream);
  if (e != cudaSuccess) return e;
  page_plan_kernel<<<1, 1024, 0, stream>>>(p);
  page_write_kernel<<<grid_for(std::min<long long>(p.page_cap, 1LL << 22) * 32, 256), 256, 0,
                      stream>>>(p);
  return cudaGetLastError();
}

}  // namespace skv
