// encode.cu -- "maps dense keys to spherical codes" (SPHERICAL KV technical
// summary 2.3) in the representation of 2.1: r~ = fp16 |k| plus per-pair
// angle and share codes, and int8 V with a per-token scale, written into the
// page row that the allocation assigned.  Also writes the dense bf16
// baseline's rows.
//
// One warp per (seq, kv head, token); lane l holds dims 4l..4l+3 (pairs 2l,
// 2l+1).  Every code is an integer decision taken exactly:
//   R2 = sum of m_c^2 over the fp16 keys (k_c = m_c 2^-24) in 128-bit integers,
//   r~ = fp16_rn(min(sqrt(double_rn(R2)) 2^-24, 65504)),
//   angle sector: quadrant from signs, binary search over fp32 boundary
//   vectors with exactly-signed fp64 cross products (no fused multiply-add),
//   share code: 16 (d/2) rho^2 > {9, 25, 49} R2 in 128-bit integers,
//   V: s = fp16_rn(absmax / 127) and rint(v / s) in IEEE fp32.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace skv {

typedef unsigned __int128 u128;

__device__ __forceinline__ uint16_t double_to_half_rn(double x) {
  uint16_t r;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(r) : "d"(x));
  return r;
}

__device__ __forceinline__ u128 warp_sum_u128(u128 v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    unsigned long long lo = (unsigned long long)v, hi = (unsigned long long)(v >> 64);
    unsigned long long olo = __shfl_xor_sync(0xFFFFFFFFu, lo, o);
    unsigned long long ohi = __shfl_xor_sync(0xFFFFFFFFu, hi, o);
    v += ((u128)ohi << 64) | olo;
  }
  return v;
}

// two fp16 (one 32-bit word) -> the two bf16 of their values, rounded to
// nearest even
__device__ __forceinline__ uint32_t half2_bits_to_bf16x2(uint32_t h) {
  const __half2 x = *reinterpret_cast<const __half2*>(&h);
  const float2 f = __half22float2(x);
  return pack_bf16x2(f.x, f.y);
}

// b-bit angle sector of the pair (x, y) = (mx, my) 2^-24 (the fp16 values as
// integers, half_bits_to_m); bxy: the 2^b boundary vectors (fp32 values held
// as doubles, (x, y) interleaved).  Within the point's quadrant q the code is
// q 2^(b-2) + (the number of the quadrant's boundaries that the point is on
// or counter-clockwise of): a prefix of them, since the side of boundary j,
// sign(bx_j y - by_j x), falls from >= 0 to < 0 once.  Each product of a
// 24-bit and an 11-bit significand is exact in fp64 and the difference is
// rounded once, so every side is exact (and unchanged by the scale 2^24).
// The count is first estimated from an fp32 arctangent of the point rotated
// into quadrant 0 (error < 2e-3 rad, against sectors of at least pi/32 rad:
// the estimate is off by at most one), then fixed by the exact sides of the
// two boundaries around it.
__device__ __forceinline__ uint32_t angle_code(long long mx, long long my, int b,
                                               const double2* bxy) {
  const double x = (double)mx, y = (double)my;
  if (x == 0.0 && y == 0.0) return 0;
  int q;
  if (x > 0 && y >= 0) q = 0;
  else if (x <= 0 && y > 0) q = 1;
  else if (x < 0 && y <= 0) q = 2;
  else q = 3;
  const int per = 1 << (b - 2);
  const int base = q * per;
  // (u, v): the point rotated by -q quarter turns, u > 0 and v >= 0
  const float fx = (float)x, fy = (float)y;
  const float u = q == 0 ? fx : (q == 1 ? fy : (q == 2 ? -fx : -fy));
  const float v = q == 0 ? fy : (q == 1 ? -fx : (q == 2 ? -fy : fx));
  const bool low = v <= u;
  const float t = low ? __fdividef(v, u) : __fdividef(u, v);  // in [0, 1]
  // atan(t) on [0, 1]: pi/4 t - t (t - 1)(0.2447 + 0.0663 t), |error| < 1.6e-3
  const float at = t * (0.78539816f - (t - 1.0f) * (0.2447f + 0.0663f * t));
  const float phi = low ? at : 1.57079633f - at;
  int lo = (int)(phi * ((float)per * 0.63661977f) + 0.5f);  // boundaries at (j + 1/2) pi / (2 per)
  lo = min(max(lo, 0), per);
  // exact sides of the boundaries lo - 1 and lo: the true count is lo - 1,
  // lo or lo + 1
  bool below = false, above = false;
  if (lo > 0) {
    const double2 c = bxy[base + lo - 1];
    below = __dsub_rn(__dmul_rn(c.x, y), __dmul_rn(c.y, x)) < 0.0;  // not yet past lo - 1
  }
  if (lo < per) {
    const double2 c = bxy[base + lo];
    above = __dsub_rn(__dmul_rn(c.x, y), __dmul_rn(c.y, x)) >= 0.0;  // already past lo
  }
  lo += above ? 1 : (below ? -1 : 0);
  return (uint32_t)(base + lo) & (uint32_t)((1 << b) - 1);
}

// 3-bit share code of the T1 variant: thresholds u > (2j + 3) / 8, j < 7,
// tested as 64 (d/2) rho^2 > (2j + 3)^2 R2; ties go to the lower code
__device__ __forceinline__ uint32_t rho_code3(long long mx, long long my, u128 R2) {
  const u128 ax = (u128)(mx < 0 ? -mx : mx), ay = (u128)(my < 0 ? -my : my);
  const u128 lhs = (ax * ax + ay * ay) * (u128)(64 * (kHeadDim / 2));
  uint32_t c = 0;
#pragma unroll
  for (int j = 0; j < 7; ++j) c += lhs > (u128)((2 * j + 3) * (2 * j + 3)) * R2;
  return c;
}

// 2-bit share code: how many thresholds u = (rho / r) sqrt(d/2) exceeds.
// Uniform grid: u > {0.75, 1.25, 1.75}, i.e. 16 (d/2) rho^2 > {9, 25, 49} R2;
// Lloyd-Max grid: u^2 > {22, 64, 145} / 64, i.e. 64 (d/2) rho^2 > {22, 64, 145} R2.
__device__ __forceinline__ uint32_t rho_code(long long mx, long long my, u128 R2, int grid) {
  const u128 ax = (u128)(mx < 0 ? -mx : mx), ay = (u128)(my < 0 ? -my : my);
  const u128 lhs = (ax * ax + ay * ay) * (u128)((grid ? 64 : 16) * (kHeadDim / 2));
  uint32_t c = 0;
  c += lhs > (u128)(grid ? 22 : 9) * R2;
  c += lhs > (u128)(grid ? 64 : 25) * R2;
  c += lhs > (u128)(grid ? 145 : 49) * R2;
  return c;
}

// byte offset, within a page's V section, of element (row, dim)
__device__ __forceinline__ int v_frag_offset(int row, int dd, int elem_bytes) {
  const int k = row >> 3, tr = row & 7, t4 = tr >> 1, lo = tr & 1;
  const int mt = dd >> 4, rem = dd & 15, g = rem & 7, hi = rem >> 3;
  const int L = 4 * g + t4, e = 2 * hi + lo;
  if (elem_bytes == 1) return k * 1024 + 512 * (mt >> 2) + 16 * L + 4 * (mt & 3) + e;
  return k * 2048 + 512 * (mt >> 1) + 16 * L + 8 * (mt & 1) + 2 * e;
}

// The boundary vectors of the three angle codes (fp32 values), in shared
// memory as doubles, (x, y) of a boundary in one 16-byte load.
struct Boundaries {
  double2 b6[64], b4[16], b5[32];
};

template <class Prm>
__device__ __forceinline__ void load_boundaries(const Prm& p, Boundaries& sb) {
  for (int i = threadIdx.x; i < 64; i += blockDim.x) {
    sb.b6[i] = make_double2(p.bx6[i], p.by6[i]);
    if (i < 32) sb.b5[i] = make_double2(p.bx5[i], p.by5[i]);
    if (i < 16) sb.b4[i] = make_double2(p.bx4[i], p.by4[i]);
  }
}

// Write one token's row `row` into `page` (tier tr, P rows): the warp's lane
// l holds the fp16 key and value components 4l..4l+3 in k4 / v4.  T0 keeps
// them (rounded to bf16 for the dense baseline and the fused T0 / bf16
// path), T1 / T2 encode them.
__device__ __forceinline__ void write_row(uint8_t* page, int P, int tr, int row, int lane,
                                          const uint16_t (&k4)[4], const uint16_t (&v4)[4],
                                          bool dense_bf16, int t1_scheme, int share_grid,
                                          const Boundaries& sb) {
  if (tr == SKV_TIER_T0) {
    uint16_t ko[4], vo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (dense_bf16) {
        ko[i] = __bfloat16_as_ushort(__float2bfloat16_rn(__half2float(__ushort_as_half(k4[i]))));
        vo[i] = __bfloat16_as_ushort(__float2bfloat16_rn(__half2float(__ushort_as_half(v4[i]))));
      } else {
        ko[i] = k4[i];
        vo[i] = v4[i];
      }
    }
    const int c = lane >> 1, e0 = (lane & 1) * 4;
    const int pos = c ^ (4 * (row & 1));
    uint2 kout;
    kout.x = (uint32_t)ko[0] | ((uint32_t)ko[1] << 16);
    kout.y = (uint32_t)ko[2] | ((uint32_t)ko[3] << 16);
    *reinterpret_cast<uint2*>(page + kHdrBytes + row * 256 + pos * 16 + e0 * 2) = kout;
    uint8_t* vsec = page + kHdrBytes + 256 * P;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint16_t*>(vsec + v_frag_offset(row, 4 * lane + i, 2)) = vo[i];
    return;
  }

  // ---- radius
  long long m[4];
  u128 sq = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = half_bits_to_m(k4[i]);
    const u128 a = (u128)(m[i] < 0 ? -m[i] : m[i]);
    sq += a * a;
  }
  const u128 R2 = warp_sum_u128(sq);
  const double r2d = u128_to_double_rn((unsigned long long)(R2 >> 64), (unsigned long long)R2);
  double r = __dmul_rn(__dsqrt_rn(r2d), 5.9604644775390625e-08);  // 2^-24
  if (r > 65504.0) r = 65504.0;
  const uint16_t rt = double_to_half_rn(r);

  // ---- codes of pairs 2 lane, 2 lane + 1
  const bool t1 = tr == SKV_TIER_T1;
  const bool v53 = t1 && t1_scheme;  // T1 variant: 5-bit angle + 3-bit share
  const int bits = t1 ? (v53 ? 5 : 6) : 4;
  const double2* bxy = t1 ? (v53 ? sb.b5 : sb.b6) : sb.b4;
  const uint32_t th0 = angle_code(m[0], m[1], bits, bxy);
  const uint32_t th1 = angle_code(m[2], m[3], bits, bxy);
  const uint32_t rh0 = v53 ? rho_code3(m[0], m[1], R2) : rho_code(m[0], m[1], R2, share_grid);
  const uint32_t rh1 = v53 ? rho_code3(m[2], m[3], R2) : rho_code(m[2], m[3], R2, share_grid);
  const uint32_t packed = th0 | (th1 << 8) | (rh0 << 16) | (rh1 << 24);
  // ---- V quantiser
  float vf[4], amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    vf[i] = __half2float(__ushort_as_half(v4[i]));
    amax = fmaxf(amax, fabsf(vf[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const __half sh = __float2half_rn(__fdiv_rn(amax, 127.0f));
  const float s = __half2float(sh);
  int8_t v8[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int c = 0;
    if (s != 0.0f) {
      c = __float2int_rn(__fdiv_rn(vf[i], s));
      c = max(-127, min(127, c));
    }
    v8[i] = (int8_t)c;
  }

  // ---- write the row
  const int cb = t1 ? 64 : 48;
  uint8_t* rsec = page + kHdrBytes;
  uint8_t* csec = rsec + 2 * P;
  uint8_t* ssec = csec + cb * P;
  uint8_t* vsec = ssec + 2 * P;
  if (lane == 0) {
    *reinterpret_cast<uint16_t*>(rsec + 2 * row) = rt;
    *reinterpret_cast<uint16_t*>(ssec + 2 * row) = __half_as_ushort(sh);
  }
  uint8_t* crow = csec + row * cb;
  if (t1) {
    // word wd (bytes 4wd..4wd+3): group g = wd / 4, j = 4 (wd % 4) + e
    uint32_t word = 0;
    const int wd = lane & 15;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int g = wd >> 2, j = 4 * (wd & 3) + e;
      const int pr = 16 * (j >> 2) + 4 * g + (j & 3);
      const uint32_t src = __shfl_sync(0xFFFFFFFFu, packed, pr >> 1);
      const uint32_t th = (src >> (8 * (pr & 1))) & 0xFFu;
      const uint32_t rh = (src >> (16 + 8 * (pr & 1))) & 0xFFu;
      word |= ((th << (v53 ? 3 : 2)) | rh) << (8 * e);
    }
    if (lane < 16) *reinterpret_cast<uint32_t*>(crow + 4 * lane) = word;
  } else {
    // words 0..7: nibbles of group g = wd / 2, j = 8 (wd % 2) + e;
    // words 8..11: crumbs of group g = wd - 8, j = e
    const int wd = lane < 12 ? lane : 0;
    const bool crumbs = wd >= 8;
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int g = crumbs ? wd - 8 : (wd >> 1);
      const int j = crumbs ? e : 8 * (wd & 1) + (e & 7);
      const int pr = 16 * (j >> 2) + 4 * g + (j & 3);
      const uint32_t src = __shfl_sync(0xFFFFFFFFu, packed, pr >> 1);
      if (crumbs) {
        const uint32_t rh = (src >> (16 + 8 * (pr & 1))) & 3u;
        word |= rh << (2 * e);
      } else if (e < 8) {
        const uint32_t th = (src >> (8 * (pr & 1))) & 15u;
        word |= th << (4 * e);
      }
    }
    if (lane < 12) *reinterpret_cast<uint32_t*>(crow + 4 * lane) = word;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) vsec[v_frag_offset(row, 4 * lane + i, 1)] = (uint8_t)v8[i];
}

// One warp per kEncodeTokens consecutive positions of a unit (block x of the
// unit's nbx blocks takes positions 8 kEncodeTokens x ..): every load of its
// tokens -- tier, row, page id, K and V -- is issued before the first row is
// written, so the dependent loads of one token overlap those of the next
// (two tokens: 14% faster than one on the 128K store; four and eight lose
// more to the registers than they gain).  One 32-bit division per block.
constexpr int kEncodeTokens = 2;

__global__ void __launch_bounds__(256) encode_kernel(const __grid_constant__ EncodeParams p,
                                                     unsigned nbx) {
  __shared__ Boundaries sb;
  load_boundaries(p, sb);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const unsigned bh = blockIdx.x / nbx;
  const long long tb =
      (long long)(blockIdx.x - bh * nbx) * (8 * kEncodeTokens) + (threadIdx.x >> 5) * kEncodeTokens;
  const int P = p.P, lp = __ffs(P) - 1;  // P is a power of two
  const long long T = min((long long)p.seq_lens[bh / (unsigned)p.Hkv], p.Tmax);
  int tr[kEncodeTokens], row[kEncodeTokens];
  long long gi[kEncodeTokens];
  uint2 kv[kEncodeTokens], vv[kEncodeTokens];
#pragma unroll
  for (int j = 0; j < kEncodeTokens; ++j) {
    const long long t = tb + j;
    const long long w = (long long)bh * p.Tmax + t;
    tr[j] = SKV_TIER_DROP;
    row[j] = 0;
    gi[j] = -1;
    if (t < T) {
      if (p.dense_bf16) {
        tr[j] = 0;
        gi[j] = (long long)p.indptr[bh] + (t >> lp);
        row[j] = (int)(t & (P - 1));
      } else {
        tr[j] = p.tier[w];
        const int loc = p.row_of[w];
        if (tr[j] < SKV_TIER_DROP && loc >= 0) {
          gi[j] = (long long)p.indptr[bh] + (loc >> lp);
          row[j] = loc & (P - 1);
        } else if (tr[j] != SKV_TIER_DROP) {
          gi[j] = -2;  // a bad tier or row: reported below
        }
      }
      kv[j] = *reinterpret_cast<const uint2*>(p.K + w * kHeadDim + 4 * lane);
      vv[j] = *reinterpret_cast<const uint2*>(p.V + w * kHeadDim + 4 * lane);
    }
  }
  uint8_t* page[kEncodeTokens];
#pragma unroll
  for (int j = 0; j < kEncodeTokens; ++j) {
    page[j] = nullptr;
    if (gi[j] >= 0 && gi[j] < p.indptr[bh + 1]) {
      const uint32_t id = p.ids[gi[j]], slot = id & 0x3FFFFFFFu;
      if ((int)(id >> 30) == tr[j] && (long long)slot < p.slots[tr[j]])
        page[j] = p.pool[tr[j]] + (long long)slot * p.stride[tr[j]];
    }
  }
#pragma unroll
  for (int j = 0; j < kEncodeTokens; ++j) {
    if (tr[j] == SKV_TIER_DROP && gi[j] == -1) continue;  // not resident (or past the sequence)
    if (!page[j]) {
      if (lane == 0) report(p.err, SKV_ERR_CORRUPT);
      continue;
    }
    const uint16_t k4[4] = {(uint16_t)(kv[j].x & 0xFFFF), (uint16_t)(kv[j].x >> 16),
                            (uint16_t)(kv[j].y & 0xFFFF), (uint16_t)(kv[j].y >> 16)};
    const uint16_t v4[4] = {(uint16_t)(vv[j].x & 0xFFFF), (uint16_t)(vv[j].x >> 16),
                            (uint16_t)(vv[j].y & 0xFFFF), (uint16_t)(vv[j].y >> 16)};
    write_row(page[j], P, tr[j], row[j], lane, k4, v4, p.dense_bf16 != 0 || p.t0_bf16 != 0,
              p.t1_scheme, p.share_grid, sb);
  }
}

// ---------------------------------------------------------------- transcode
// Re-tiering's data step, one warp per resident token of a rewritten page
// (a page at or after its segment's first change).  Its old row is either
// T0 -- the exact fp16 K and V, read back from the old page in the T0 row
// order and written (T0) or encoded (T1 / T2) as the encode does from dense
// inputs -- or T1 / T2 of the same tier, whose radius, code row, scale and
// int8 V are copied (the V fragment order depends on the row index).

// the page of row `loc` of unit u in a page table, or null when it is not
// a page of tier tr in range
__device__ __forceinline__ uint8_t* row_page(const TranscodeParams& p, const int32_t* indptr,
                                             const uint32_t* ids, long long u, int tr, int loc) {
  if (loc < 0) return nullptr;
  const long long gi = (long long)indptr[u] + loc / p.P;
  if (gi >= indptr[u + 1] || gi < 0 || gi >= p.page_cap) return nullptr;
  const uint32_t id = ids[gi], slot = id & 0x3FFFFFFFu;
  if ((int)(id >> 30) != tr || (long long)slot >= p.slots[tr]) return nullptr;
  return p.pool[tr] + (long long)slot * p.stride[tr];
}

// First pass, one thread per (unit, position): the resident rows that lie in
// rewritten pages (at or after their segment's first change) go to a list
// (one atomic per warp).  Most rows are in kept pages, so the second pass
// runs over few rows.
__global__ void __launch_bounds__(256) transcode_list_kernel(const __grid_constant__ TranscodeParams p,
                                                             unsigned nbx) {
  const unsigned u = blockIdx.x / nbx;
  const long long t = (long long)(blockIdx.x - u * nbx) * blockDim.x + threadIdx.x;
  bool need = false;
  long long w = 0;
  if (t < p.Tmax && t < p.seq_lens[u / (unsigned)p.Hkv]) {
    w = (long long)u * p.Tmax + t;
    const int tn = p.tier[w];
    if (tn < SKV_TIER_DROP) {
      const int rn = p.row_of[w];
      need = rn < 0 ||
             rn / p.P - (p.tier_indptr[3 * u + tn] - p.indptr[u]) >= p.keep[3 * u + tn];
    }
  }
  const unsigned mask = __ballot_sync(0xFFFFFFFFu, need);
  if (!mask) return;
  const int lane = threadIdx.x & 31, leader = __ffs(mask) - 1;
  unsigned long long base = 0;
  if (lane == leader) base = atomicAdd(p.count, (unsigned long long)__popc(mask));
  base = __shfl_sync(0xFFFFFFFFu, base, leader);
  if (need) p.list[base + __popc(mask & ((1u << lane) - 1))] = (uint32_t)w;
}

// Second pass, a warp per listed row (a grid-stride loop): its old row is
// either T0 -- the exact fp16 K and V, read back from the old page in the T0
// row order and written (T0) or encoded (T1 / T2) as the encode does from
// dense inputs -- or T1 / T2 of the same tier, whose radius, code row, scale
// and int8 V are copied (the V fragment order depends on the row index).
__global__ void __launch_bounds__(256) transcode_kernel(const __grid_constant__ TranscodeParams p) {
  __shared__ Boundaries sb;
  load_boundaries(p, sb);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const long long n = (long long)*p.count;
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n; i += nwarps) {
    const long long w = p.list[i];
    const long long u = w / p.Tmax;
    const int tn = p.tier[w];
    const int rn = p.row_of[w], P = p.P;
    const int to = p.tier_old[w], ro = to < SKV_TIER_DROP ? p.row_old[w] : -1;
    uint8_t* dst = row_page(p, p.indptr, p.ids, u, tn, rn);
    const uint8_t* src = to < SKV_TIER_DROP ? row_page(p, p.indptr_old, p.ids_old, u, to, ro)
                                            : nullptr;
    if (!dst || !src || (to != SKV_TIER_T0 && to != tn)) {
      if (lane == 0) report(p.err, SKV_ERR_CORRUPT);
      continue;
    }
    const int r_new = rn % P, r_old = ro % P;
    if (to == SKV_TIER_T0) {
      const int c = lane >> 1;
      const uint2 kv = *reinterpret_cast<const uint2*>(
          src + kHdrBytes + r_old * 256 + (c ^ (4 * (r_old & 1))) * 16 + (lane & 1) * 8);
      const uint8_t* vsec = src + kHdrBytes + 256 * P;
      uint16_t k4[4] = {(uint16_t)(kv.x & 0xFFFF), (uint16_t)(kv.x >> 16),
                        (uint16_t)(kv.y & 0xFFFF), (uint16_t)(kv.y >> 16)};
      uint16_t v4[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        v4[k] = *reinterpret_cast<const uint16_t*>(vsec + v_frag_offset(r_old, 4 * lane + k, 2));
      write_row(dst, P, tn, r_new, lane, k4, v4, false, p.t1_scheme, p.share_grid, sb);
      continue;
    }
    // T1 / T2 row: r~ (fp16 [P]), codes ([P][cb]), scale (fp16 [P]), int8 V
    const int cb = tn == SKV_TIER_T1 ? 64 : 48;
    const uint8_t* rs = src + kHdrBytes;
    uint8_t* rd = dst + kHdrBytes;
    if (lane == 0) {
      *reinterpret_cast<uint16_t*>(rd + 2 * r_new) =
          *reinterpret_cast<const uint16_t*>(rs + 2 * r_old);
      *reinterpret_cast<uint16_t*>(rd + (2 + cb) * P + 2 * r_new) =
          *reinterpret_cast<const uint16_t*>(rs + (2 + cb) * P + 2 * r_old);
    }
    if (lane < cb / 4)
      *reinterpret_cast<uint32_t*>(rd + 2 * P + cb * r_new + 4 * lane) =
          *reinterpret_cast<const uint32_t*>(rs + 2 * P + cb * r_old + 4 * lane);
    const uint8_t* vs = rs + (4 + cb) * P;
    uint8_t* vd = rd + (4 + cb) * P;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      vd[v_frag_offset(r_new, 4 * lane + k, 1)] = vs[v_frag_offset(r_old, 4 * lane + k, 1)];
  }
}

// ------------------------------------------------------------------ append
// Decode-time ingest (the step before the decode in a serving loop): the
// token at position t = seq_lens[b] of every kv head h becomes resident as
// T0, the newest token being in the protected recent window.  It goes into
// the next row of its unit's last T0 page, or, when that page is full or
// the unit has none, into a new T0 page (a slot from the T0 free list)
// inserted at the end of the unit's T0 segment; the later page ids move up
// and the T1/T2 rows of that unit move one page down (row_of += P).  The
// result is the layout a fresh pack of the same tiers gives (page slots
// aside).  Three kernels: plan (one block: per-unit decisions, a scan of the
// new pages, the new CSR offsets), move (page ids to their new positions,
// the new ids and the row map of a unit that gained a page; idle unless a
// page is added) and write (the token's row, headers, tier and row_of).

__global__ void __launch_bounds__(1024) append_plan_kernel(const __grid_constant__ AppendParams p) {
  __shared__ int scan[1024];
  __shared__ int bad;
  const int U = p.B * p.Hkv;
  const AppendWs wl = append_ws(U, p.page_cap);
  int32_t* const ws = p.ws;
  const int tid = threadIdx.x, nt = blockDim.x;
  if (tid == 0) bad = 0;
  __syncthreads();
  // per unit: the token's position and whether a new T0 page is needed
  const int per = (U + nt - 1) / nt;
  const int ua = min(U, tid * per), ub = min(U, ua + per);
  int cnt = 0;
  for (int u = ua; u < ub; ++u) {
    const int t = p.seq_lens[u / p.Hkv];
    const int A0 = p.tier_indptr[3 * u], A1 = p.tier_indptr[3 * u + 1];
    int need = 1;
    if (t < 0 || (long long)t >= p.Tmax) atomicExch(&bad, SKV_ERR_ARG);
    if (A1 > A0) {
      const uint32_t id = p.ids[A1 - 1];
      const uint32_t slot = id & 0x3FFFFFFFu;
      if ((id >> 30) != 0u || (long long)slot >= p.slots0) {
        atomicExch(&bad, SKV_ERR_CORRUPT);
      } else {
        const uint32_t cnt_rows = *reinterpret_cast<const uint16_t*>(p.pool0 + (long long)slot * p.stride0);
        need = cnt_rows >= (uint32_t)p.P;
      }
    }
    ws[wl.t + u] = t;
    ws[wl.need + u] = need;
    ws[wl.a1 + u] = A1;
    cnt += need;
  }
  // exclusive scan of the new pages over the units
  scan[tid] = cnt;
  __syncthreads();
  for (int o = 1; o < nt; o <<= 1) {
    const int v = tid >= o ? scan[tid - o] : 0;
    __syncthreads();
    scan[tid] += v;
    __syncthreads();
  }
  const int total = scan[nt - 1];
  int before = scan[tid] - cnt;
  for (int u = ua; u < ub; ++u) {
    ws[wl.nb + u] = before;
    before += ws[wl.need + u];
  }
  const int n_raw = p.indptr[U];
  const int n_old = max(0, (int)min((long long)n_raw, p.page_cap));
  const int cur = *p.free0_cursor;
  if (tid == 0) {
    if (n_raw < 0 || (long long)n_raw > p.page_cap || cur < 0) atomicExch(&bad, SKV_ERR_CORRUPT);
    else if ((long long)n_old + total > p.page_cap || (long long)cur + total > p.free0_len)
      atomicExch(&bad, SKV_ERR_POOL);
  }
  if (total > 0) {  // the page ids move only when pages are added
    for (int g = tid; g < n_old; g += nt) ws[wl.oids + g] = (int32_t)p.ids[g];
    for (int u = tid; u <= U; u += nt) ws[wl.oindptr + u] = p.indptr[u];
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      report(p.err, bad);
      ws[wl.flag] = 1;
    }
    return;
  }
  // the new offsets (every read of the old ones is above the barrier)
  for (int u = ua; u < ub; ++u) {
    const int nb = ws[wl.nb + u], need = ws[wl.need + u];
    p.indptr[u] += nb;
    p.tier_indptr[3 * u] += nb;
    p.tier_indptr[3 * u + 1] += nb + need;
    p.tier_indptr[3 * u + 2] += nb + need;
  }
  for (int b = tid; b < p.B; b += nt) p.seq_lens[b] += 1;
  if (tid == 0) {
    p.indptr[U] += total;
    p.tier_indptr[3 * U] += total;
    ws[wl.flag] = 0;
    ws[wl.cur] = cur;
    ws[wl.total] = total;
    *p.free0_cursor = cur + total;
  }
}

// When pages are added: old page g to its new position (its unit found by
// binary search over the old offsets), each unit's new id, and, for a unit
// that gained a T0 page, its T1/T2 rows one page further down the list (the
// three are independent).  One small grid-stride launch that leaves at once
// on the steps that add no page.
__global__ void __launch_bounds__(256) append_move_kernel(const __grid_constant__ AppendParams p) {
  const int U = p.B * p.Hkv;
  const AppendWs wl = append_ws(U, p.page_cap);
  const int32_t* const ws = p.ws;
  if (ws[wl.flag] || ws[wl.total] == 0) return;
  const long long nthr = (long long)gridDim.x * blockDim.x;
  const long long i0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int n_old = ws[wl.oindptr + U];
  for (long long g = i0; g < n_old; g += nthr) {
    int lo = 0, hi = U - 1;  // the unit u with oindptr[u] <= g < oindptr[u + 1]
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (ws[wl.oindptr + mid] <= g) lo = mid; else hi = mid - 1;
    }
    const int u = lo;
    const long long shift = ws[wl.nb + u] + (g >= ws[wl.a1 + u] ? ws[wl.need + u] : 0);
    p.ids[g + shift] = (uint32_t)ws[wl.oids + g];
  }
  for (long long u = i0; u < U; u += nthr) {
    if (!ws[wl.need + u]) continue;
    const int nb = ws[wl.nb + u];
    const uint32_t slot = p.free0[ws[wl.cur] + nb];
    if ((long long)slot >= p.slots0) report(p.err, SKV_ERR_POOL);
    p.ids[ws[wl.a1 + u] + nb] = slot & 0x3FFFFFFFu;  // tier 0
  }
  const long long n = (long long)U * p.Tmax;
  for (long long i = i0; i < n; i += nthr) {
    const long long u = i / p.Tmax, k = i - u * p.Tmax;
    if (!ws[wl.need + u] || k >= ws[wl.t + u]) continue;
    const uint8_t tr = p.tier[i];
    if (tr == SKV_TIER_T1 || tr == SKV_TIER_T2) p.row_of[i] += p.P;
  }
}

// a warp per unit: the new page (zeroed, header) or the next row of the last
// T0 page, the token's fp16 K and V in the T0 row order, tier and row_of
__global__ void __launch_bounds__(256) append_write_kernel(const __grid_constant__ AppendParams p) {
  const int U = p.B * p.Hkv;
  const AppendWs wl = append_ws(U, p.page_cap);
  const int32_t* const ws = p.ws;
  const int u = (int)(((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (u >= U || ws[wl.flag]) return;
  const int b = u / p.Hkv, h = u % p.Hkv, P = p.P;
  const int t = ws[wl.t + u], need = ws[wl.need + u];
  const int first = p.tier_indptr[3 * u], t0end = p.tier_indptr[3 * u + 1];
  const uint32_t id = p.ids[t0end - 1];
  const uint32_t slot = id & 0x3FFFFFFFu;
  if ((id >> 30) != 0u || (long long)slot >= p.slots0) {
    if (lane == 0) report(p.err, SKV_ERR_CORRUPT);
    return;
  }
  uint8_t* page = p.pool0 + (long long)slot * p.stride0;
  int row;
  if (need) {
    const int payload = kHdrBytes + P * 512;
    for (int o = 16 * lane; o < payload; o += 512) *reinterpret_cast<uint4*>(page + o) = make_uint4(0, 0, 0, 0);
    __syncwarp();
    if (lane == 0)
      *reinterpret_cast<uint4*>(page) =
          make_uint4(1u | ((uint32_t)SKV_TIER_T0 << 16) | ((uint32_t)kPageMagic << 24), (uint32_t)b,
                     (uint32_t)h, (uint32_t)(t0end - 1 - first));
    row = 0;
  } else {
    uint32_t c = 0;
    if (lane == 0) {
      c = *reinterpret_cast<const uint16_t*>(page);
      *reinterpret_cast<uint16_t*>(page) = (uint16_t)(c + 1);
    }
    row = (int)__shfl_sync(0xFFFFFFFFu, c, 0);
  }
  __syncwarp();
  // the row, as the pack lays out T0 rows (see encode_kernel), in bf16 for
  // the fused T0 / bf16 path
  const long long w = (long long)u * kHeadDim;
  uint2 kv = *reinterpret_cast<const uint2*>(p.K + w + 4 * lane);
  uint2 vv = *reinterpret_cast<const uint2*>(p.V + w + 4 * lane);
  if (p.t0_bf16) {
    kv = make_uint2(half2_bits_to_bf16x2(kv.x), half2_bits_to_bf16x2(kv.y));
    vv = make_uint2(half2_bits_to_bf16x2(vv.x), half2_bits_to_bf16x2(vv.y));
  }
  const int c = lane >> 1, e0 = (lane & 1) * 4;
  const int pos = c ^ (4 * (row & 1));
  *reinterpret_cast<uint2*>(page + kHdrBytes + row * 256 + pos * 16 + e0 * 2) = kv;
  uint8_t* vsec = page + kHdrBytes + 256 * P;
  const uint16_t v4[4] = {(uint16_t)(vv.x & 0xFFFF), (uint16_t)(vv.x >> 16),
                          (uint16_t)(vv.y & 0xFFFF), (uint16_t)(vv.y >> 16)};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<uint16_t*>(vsec + v_frag_offset(row, 4 * lane + i, 2)) = v4[i];
  // tier and row map: the token; with a new page, the unit's T1/T2 rows
  // follow it one page further down the list
  const long long base = (long long)u * p.Tmax;
  if (lane == 0) {
    p.tier[base + t] = SKV_TIER_T0;
    p.row_of[base + t] = (t0end - 1 - first) * P + row;
  }
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  const int U = p.B * p.Hkv;
  if (U == 0) return cudaSuccess;
  append_plan_kernel<<<1, 1024, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // two blocks per SM, leaving at once when no page is added
  append_move_kernel<<<296, 256, 0, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  append_write_kernel<<<(unsigned)((U + 7) / 8), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_transcode(const TranscodeParams& p, cudaStream_t stream) {
  const long long U = (long long)p.B * p.Hkv;
  if (U == 0 || p.Tmax == 0) return cudaSuccess;
  const long long nbx = (p.Tmax + 255) / 256;
  if (U * nbx > 0x7FFFFFFFLL || U * p.Tmax > 0xFFFFFFFFLL) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(p.count, 0, sizeof(unsigned long long), stream);
  if (e != cudaSuccess) return e;
  transcode_list_kernel<<<(unsigned)(U * nbx), 256, 0, stream>>>(p, (unsigned)nbx);
  // a few resident blocks per SM loop over the listed rows
  transcode_kernel<<<148 * 4, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_encode(const EncodeParams& p, cudaStream_t stream) {
  const long long U = (long long)p.B * p.Hkv;
  if (U == 0 || p.Tmax == 0) return cudaSuccess;
  const long long nbx = (p.Tmax + 8 * kEncodeTokens - 1) / (8 * kEncodeTokens);
  if (U * nbx > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  encode_kernel<<<(unsigned)(U * nbx), 256, 0, stream>>>(p, (unsigned)nbx);
  return cudaGetLastError();
}

}  // namespace skv
