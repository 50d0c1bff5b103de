// decode.cu -- ADA paged decode (SPHERICAL KV technical summary 2.1: logits
// computed directly from the radius and angle codes, no dense key
// materialised; 2.2: tier-homogeneous pages read in one header-guided pass)
// and the dense bf16 paged-decode baseline built on the same skeleton.
//
// Work split ("split-K over pages"): the CSR page list of all units
// (unit = (seq, kv head)) is one array of N pages; CTA c streams the run
// [floor(c N / S), floor((c+1) N / S)) and emits one partial (m, l, o) per
// unit it touches, at partial slot c + u.  A merge kernel combines them.
//
// CTA = 8 consumer warps + 1 producer warp.  The producer copies whole
// pages (header included) with 1-D bulk async copies into a byte ring in
// shared memory, 64 tokens per "item" (64/P pages), tracked by full/empty
// mbarriers; consumer warp w takes rows [8w, 8w+8) of each item.
//
// Consumer lane map: lane = 4 t + g, t = token of the 8-row group, g = pair
// group.  Logits: lane (t, g) sums 16 pairs (T1/T2, LUT gathers from shared
// memory) or 32 dims (T0) for all G query heads of the group, then a 4-lane
// reduce-scatter leaves head g's logit in lane (t, g).  P.V: mma.sync
// m16n8k8, A = V^T fragment read straight from the page (the page stores V
// in fragment order), B = P (8 tokens x 8 heads, zero-padded), f32 accum.
#include "common.cuh"
#include "kernels.h"

namespace skv {

constexpr int kNCW = 8;
constexpr int kDecodeThreads = (kNCW + 1) * 32;
constexpr int kNSlot = 16;
constexpr int kMaxIPP = 4;
constexpr uint32_t kInvalidOff = 0xFFFFFFFFu;

template <int G, bool DENSE>
struct __align__(16) DecodeSmem {
  unsigned long long full[kNSlot];
  unsigned long long empty[kNSlot];
  uint32_t item_off[kNSlot][kMaxIPP];
  uint32_t item_np[kNSlot];
  uint32_t item_tier[kNSlot];          // byte k = tier of page k
  long long item_start[kNSlot];         // producer bookkeeping (ring position)
  int abort_flag;
  int pad_[3];
  float ml[kNCW][4][2];
  float O[4][kHeadDim];
  float q32[4][kHeadDim];
  uint16_t q16[4][kHeadDim];            // fp16 (ADA T0) or bf16 (dense) bits
  uint16_t lut1[DENSE ? 8 : 64 * kPairs * G];   // [code 64][pair 64][G] fp16
  uint16_t lut2[DENSE ? 8 : 16 * kPairs * G];   // [code 16][pair 64][G] fp16
};

__device__ __forceinline__ long long chunk_begin(int c, long long N, int S) {
  return (long long)c * N / S;
}

// share level (code + 1) / 16 as fp16 bits: 0x2C00, 0x3000, 0x3200, 0x3400
__device__ __forceinline__ uint16_t rho_half(uint32_t rh) {
  return (uint16_t)__byte_perm(0x30002C00u, 0x34003200u, rh * 0x22u + 0x10u);
}

template <int G>
__device__ __forceinline__ void lut_gather(const uint16_t* e, uint16_t rho, float (&s)[G]) {
  if constexpr (G == 4) {
    uint2 v = *reinterpret_cast<const uint2*>(e);
    s[0] = fma_f16f16f32(rho, (uint16_t)(v.x & 0xFFFF), s[0]);
    s[1] = fma_f16f16f32(rho, (uint16_t)(v.x >> 16), s[1]);
    s[2] = fma_f16f16f32(rho, (uint16_t)(v.y & 0xFFFF), s[2]);
    s[3] = fma_f16f16f32(rho, (uint16_t)(v.y >> 16), s[3]);
  } else if constexpr (G == 2) {
    uint32_t v = *reinterpret_cast<const uint32_t*>(e);
    s[0] = fma_f16f16f32(rho, (uint16_t)(v & 0xFFFF), s[0]);
    s[1] = fma_f16f16f32(rho, (uint16_t)(v >> 16), s[1]);
  } else {
    s[0] = fma_f16f16f32(rho, *e, s[0]);
  }
}

// Per-lane partial logits of token `row` for the T1 page at pg.
template <int G>
__device__ __forceinline__ void logits_t1(const uint8_t* pg, int P, int row, int g,
                                          const uint16_t* lut1, float (&s)[G]) {
  const uint8_t* cd = pg + kHdrBytes + 2 * P;
  uint4 cw = *reinterpret_cast<const uint4*>(cd + row * 64 + 16 * g);
  const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
  const uint32_t x3 = row & 3;
  // element (code th, pair 4*(j ^ x3) + g) sits at lut1 + (th*64 + pair)*G
  const uint16_t* base = lut1 + g * G;
  uint32_t xo[4];
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) xo[jj] = ((uint32_t)jj ^ x3) * 4 * G;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    uint32_t byte = (w[j >> 2] >> (8 * (j & 3))) & 0xFFu;
    uint32_t th = byte >> 2;
    const uint16_t* e = base + (j & ~3) * 4 * G + xo[j & 3] + th * (kPairs * G);
    lut_gather<G>(e, rho_half(byte & 3u), s);
  }
}

template <int G>
__device__ __forceinline__ void logits_t2(const uint8_t* pg, int P, int row, int g,
                                          const uint16_t* lut2, float (&s)[G]) {
  const uint8_t* cd = pg + kHdrBytes + 2 * P + row * 48;
  uint2 nw = *reinterpret_cast<const uint2*>(cd + 8 * g);
  uint32_t cr = *reinterpret_cast<const uint32_t*>(cd + 32 + 4 * g);
  const uint32_t x3 = row & 3;
  const uint16_t* base = lut2 + g * G;
  uint32_t xo[4];
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) xo[jj] = ((uint32_t)jj ^ x3) * 4 * G;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    uint32_t word = (j < 8) ? nw.x : nw.y;
    uint32_t th = (word >> (4 * (j & 7))) & 15u;
    uint32_t rh = (cr >> (2 * j)) & 3u;
    const uint16_t* e = base + (j & ~3) * 4 * G + xo[j & 3] + th * (kPairs * G);
    lut_gather<G>(e, rho_half(rh), s);
  }
}

// T0 (fp16 K) or dense (bf16 K): lane (t, g) covers dims 8c..8c+7 for the
// chunks c = 4i + g, stored at chunk position c ^ 4(row & 1).
template <int G, bool BF16>
__device__ __forceinline__ void logits_dense(const uint8_t* pg, int row, int g,
                                             const uint16_t (*q16)[kHeadDim], float (&s)[G]) {
  const uint8_t* krow = pg + kHdrBytes + row * 256;
  const uint32_t sw = 4u * (row & 1);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t c = 4 * i + g;
    uint4 kc = *reinterpret_cast<const uint4*>(krow + ((c ^ sw) * 16));
    const uint32_t kw[4] = {kc.x, kc.y, kc.z, kc.w};
#pragma unroll
    for (int h = 0; h < G; ++h) {
      uint4 qc = *reinterpret_cast<const uint4*>(&q16[h][8 * c]);
      const uint32_t qw[4] = {qc.x, qc.y, qc.z, qc.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if constexpr (BF16) {
          s[h] = fma_bf16bf16f32((uint16_t)(kw[e] & 0xFFFF), (uint16_t)(qw[e] & 0xFFFF), s[h]);
          s[h] = fma_bf16bf16f32((uint16_t)(kw[e] >> 16), (uint16_t)(qw[e] >> 16), s[h]);
        } else {
          s[h] = fma_f16f16f32((uint16_t)(kw[e] & 0xFFFF), (uint16_t)(qw[e] & 0xFFFF), s[h]);
          s[h] = fma_f16f16f32((uint16_t)(kw[e] >> 16), (uint16_t)(qw[e] >> 16), s[h]);
        }
      }
    }
  }
}

// 4-lane reduce-scatter: afterwards lane g holds the full sum of head g % G.
template <int G>
__device__ __forceinline__ float reduce_scatter(float (&s)[G], int g) {
  if constexpr (G == 4) {
    const bool up = (g & 2) != 0;
    float x0 = __shfl_xor_sync(0xFFFFFFFFu, up ? s[0] : s[2], 2);
    float x1 = __shfl_xor_sync(0xFFFFFFFFu, up ? s[1] : s[3], 2);
    float a0 = (up ? s[2] : s[0]) + x0;
    float a1 = (up ? s[3] : s[1]) + x1;
    const bool odd = (g & 1) != 0;
    float y = __shfl_xor_sync(0xFFFFFFFFu, odd ? a0 : a1, 1);
    return (odd ? a1 : a0) + y;
  } else if constexpr (G == 2) {
    s[0] += __shfl_xor_sync(0xFFFFFFFFu, s[0], 2);
    s[1] += __shfl_xor_sync(0xFFFFFFFFu, s[1], 2);
    const bool odd = (g & 1) != 0;
    float y = __shfl_xor_sync(0xFFFFFFFFu, odd ? s[0] : s[1], 1);
    return (odd ? s[1] : s[0]) + y;
  } else {
    float a = s[0];
    a += __shfl_xor_sync(0xFFFFFFFFu, a, 2);
    a += __shfl_xor_sync(0xFFFFFFFFu, a, 1);
    return a;
  }
}

struct WarpState {
  float m;         // running max (log2 domain) of head g % G
  float l;         // partial denominator of (token slot t, head g % G)
  float acc[8][4];  // O^T fragments: [m-tile][c0..c3]
};

// Online softmax of one 8-token chunk and P.V into the accumulators.
// logit: log2-domain logit of (token t, head g % G) or -inf.
// VK: 0 int8 V (1 KB group block), 1 fp16 V (2 KB), 2 bf16 V (2 KB).
template <int G, int VK>
__device__ __forceinline__ void softmax_pv(float logit, float vscale, const uint8_t* vblock,
                                           WarpState& st, int lane) {
  float cm = logit;
  cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 4));
  cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 8));
  cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 16));
  const float m_new = fmaxf(st.m, cm);
  const bool fin = m_new != -INFINITY;
  const float alpha = (fin && st.m != m_new) ? exp2f(st.m - m_new) : 1.0f;
  const float p = (logit != -INFINITY) ? exp2f(logit - m_new) : 0.0f;
  st.l = st.l * alpha + p;
  st.m = m_new;
  const int gq = lane >> 2, t4 = lane & 3;
  if (__any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
    const int n0 = 2 * t4, n1 = 2 * t4 + 1;
    float a0 = __shfl_sync(0xFFFFFFFFu, alpha, n0 < G ? n0 : 0);
    float a1 = __shfl_sync(0xFFFFFFFFu, alpha, n1 < G ? n1 : 0);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      st.acc[mt][0] *= a0;
      st.acc[mt][1] *= a1;
      st.acc[mt][2] *= a0;
      st.acc[mt][3] *= a1;
    }
  }
  const float pp = p * vscale;
  // B fragment: (k = tokens 2 t4, 2 t4 + 1; n = head gq), zero for gq >= G
  const int src = 8 * t4 + (gq < G ? gq : 0);
  float b0 = __shfl_sync(0xFFFFFFFFu, pp, src);
  float b1 = __shfl_sync(0xFFFFFFFFu, pp, src + 4);
  if (gq >= G) {
    b0 = 0.0f;
    b1 = 0.0f;
  }
  if constexpr (VK == 0) {
    const uint32_t bf = pack_f16x2(b0, b1);
    uint4 x = *reinterpret_cast<const uint4*>(vblock + lane * 16);
    uint4 y = *reinterpret_cast<const uint4*>(vblock + 512 + lane * 16);
    const uint32_t vw[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t a0, a1;
      s8x4_to_f16x2x2(vw[mt], a0, a1);
      mma_16816_f16(st.acc[mt], a0, a1, bf);
    }
  } else {
    const uint32_t bf = (VK == 1) ? pack_f16x2(b0, b1) : pack_bf16x2(b0, b1);
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
      uint4 z = *reinterpret_cast<const uint4*>(vblock + qq * 512 + lane * 16);
      if constexpr (VK == 1) {
        mma_16816_f16(st.acc[2 * qq], z.x, z.y, bf);
        mma_16816_f16(st.acc[2 * qq + 1], z.z, z.w, bf);
      } else {
        mma_16816_bf16(st.acc[2 * qq], z.x, z.y, bf);
        mma_16816_bf16(st.acc[2 * qq + 1], z.z, z.w, bf);
      }
    }
  }
}

template <int G, bool DENSE>
__device__ __forceinline__ void process_rows(const DecodeParams& p, DecodeSmem<G, DENSE>& sm,
                                             const uint8_t* pg, uint32_t tier, int row0,
                                             WarpState& st, int lane) {
  const int t = lane >> 2, g = lane & 3;
  const int P = p.P;
  const uint32_t cnt = *reinterpret_cast<const uint16_t*>(pg);
  const uint32_t htier = pg[2];
  const uint32_t magic = pg[3];
  if (htier != tier || magic != kPageMagic || cnt > (uint32_t)P) {
    if (lane == 0) report(p.err, SKV_ERR_CORRUPT);
    return;
  }
  if ((uint32_t)row0 >= cnt) return;
  const int row = row0 + t;
  const bool valid = (uint32_t)row < cnt;
  float s[G];
#pragma unroll
  for (int h = 0; h < G; ++h) s[h] = 0.0f;
  if constexpr (DENSE) {
    logits_dense<G, true>(pg, row, g, sm.q16, s);
    float r = reduce_scatter<G>(s, g);
    float logit = valid ? r * p.qk_scale_log2 : -INFINITY;
    softmax_pv<G, 2>(logit, 1.0f, pg + kHdrBytes + 256 * P + (row0 >> 3) * 2048, st, lane);
  } else {
    if (tier == SKV_TIER_T0) {
      logits_dense<G, false>(pg, row, g, sm.q16, s);
      float r = reduce_scatter<G>(s, g);
      float logit = valid ? r * p.qk_scale_log2 : -INFINITY;
      softmax_pv<G, 1>(logit, 1.0f, pg + kHdrBytes + 256 * P + (row0 >> 3) * 2048, st, lane);
    } else {
      const bool t1 = tier == SKV_TIER_T1;
      if (t1)
        logits_t1<G>(pg, P, row, g, sm.lut1, s);
      else
        logits_t2<G>(pg, P, row, g, sm.lut2, s);
      float r = reduce_scatter<G>(s, g);
      const uint16_t* rt = reinterpret_cast<const uint16_t*>(pg + kHdrBytes);
      const int cb = t1 ? 64 : 48;
      const uint16_t* sc = reinterpret_cast<const uint16_t*>(pg + kHdrBytes + 2 * P + cb * P);
      const float rtil = __half2float(__ushort_as_half(rt[row]));
      const float vs = __half2float(__ushort_as_half(sc[row]));
      float logit = valid ? r * (rtil * p.qk_scale_log2) : -INFINITY;
      const uint8_t* vsec = pg + kHdrBytes + (2 + cb + 2) * P;
      softmax_pv<G, 0>(logit, valid ? vs : 0.0f, vsec + (row0 >> 3) * 1024, st, lane);
    }
  }
}

template <int G, bool DENSE>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    decode_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  using Smem = DecodeSmem<G, DENSE>;
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  uint8_t* ring = smem_raw + ((sizeof(Smem) + 127) / 128) * 128;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const int U = p.B * p.Hkv;
  const long long N = p.indptr[U];
  const long long g0 = chunk_begin(c, N, p.S), g1 = chunk_begin(c + 1, N, p.S);
  const int ipp = 64 >> p.log2P;

  if (tid == 0) {
    for (int i = 0; i < kNSlot; ++i) {
      mbar_init(smem_u32(&sm.full[i]), 1);
      mbar_init(smem_u32(&sm.empty[i]), kNCW);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (g0 >= g1) return;

  // first unit whose pages reach past g0: largest u with indptr[u] <= g0
  int lo = 0, hi = U;
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (p.indptr[mid] <= g0) lo = mid; else hi = mid;
  }
  const int u0 = lo;

  if (warp == kNCW) {
    // ------------------------------------------------------------ producer
    const uint32_t R = (uint32_t)p.ring_bytes;
    long long head = 0;
    int it = 0, tail = 0;
    long long wbase = -1;  // first page of the id window held in lanes
    uint32_t idwin = 0;
    bool ok = true;
    for (int u = u0; u < U && ok; ++u) {
      const long long iu0 = p.indptr[u], iu1 = p.indptr[u + 1];
      if (iu0 >= g1) break;
      const long long a = max(g0, iu0), b = min(g1, iu1);
      for (long long pg = a; pg < b && ok; pg += ipp) {
        const int n = (int)min((long long)ipp, b - pg);
        uint32_t sizes[kMaxIPP], ids[kMaxIPP];
        uint32_t total = 0;
#pragma unroll
        for (int k = 0; k < kMaxIPP; ++k) {
          sizes[k] = 0;
          ids[k] = 0;
          if (k < n) {
            const long long gp = pg + k;
            if (wbase < 0 || gp >= wbase + 32) {
              wbase = gp;
              idwin = (gp + lane < g1) ? p.ids[gp + lane] : 0u;
            }
            const uint32_t id = __shfl_sync(0xFFFFFFFFu, idwin, (int)(gp - wbase));
            const uint32_t tr = id >> 30, slot = id & 0x3FFFFFFFu;
            ids[k] = id;
            const bool valid = DENSE ? (tr == 0 && slot < (uint64_t)p.slots[0])
                                     : (tr < 3 && slot < (uint64_t)p.slots[tr]);
            if (valid) sizes[k] = (uint32_t)p.payload[tr];
            else if (lane == 0) report(p.err, SKV_ERR_CORRUPT);
            total += sizes[k];
          }
        }
        if (lane == 0) {
          const int s = it % kNSlot;
          long long pos = head;
          uint32_t off = (uint32_t)(pos % R);
          if (off + total > R) {
            pos += R - off;
            off = 0;
          }
          while (tail < it && (it - tail >= kNSlot ||
                               sm.item_start[tail % kNSlot] < pos + (long long)total - R)) {
            if (!mbar_wait_bounded(smem_u32(&sm.empty[tail % kNSlot]),
                                   (uint32_t)((tail / kNSlot) & 1), &sm.abort_flag)) {
              ok = false;
              break;
            }
            ++tail;
          }
          if (ok) {
            sm.item_start[s] = pos;
            sm.item_np[s] = (uint32_t)n;
            uint32_t o = off, tiers = 0;
            for (int k = 0; k < n; ++k) {
              sm.item_off[s][k] = sizes[k] ? o : kInvalidOff;
              tiers |= (ids[k] >> 30) << (8 * k);
              o += sizes[k];
            }
            sm.item_tier[s] = tiers;
            const uint32_t full = smem_u32(&sm.full[s]);
            mbar_arrive_expect_tx(full, total);
            o = off;
            for (int k = 0; k < n; ++k) {
              if (sizes[k]) {
                const uint32_t tr = ids[k] >> 30, slot = ids[k] & 0x3FFFFFFFu;
                bulk_g2s(smem_u32(ring + o), p.pool[tr] + (long long)slot * p.stride[tr], sizes[k],
                         full);
                o += sizes[k];
              }
            }
            head = pos + total;
            ++it;
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
        it = __shfl_sync(0xFFFFFFFFu, it, 0);
      }
    }
    if (lane == 0 && !ok) {
      report(p.err, SKV_ERR_TIMEOUT);
      sm.abort_flag = 1;
      // let every copy already issued land before the CTA can exit
      for (int j = max(0, it - kNSlot); j < it; ++j) {
        long long t0 = clock64();
        while (!mbar_try_wait(smem_u32(&sm.full[j % kNSlot]), (uint32_t)((j / kNSlot) & 1)) &&
               clock64() - t0 < kWaitLimitCycles) {
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int nct = kNCW * 32;
  const int t4 = lane & 3, gq = lane >> 2;
  // A failed (timed-out) wait never breaks the loops: every consumer warp
  // must run the same sequence of named barriers.  After a failure the CTA's
  // abort flag makes every later wait return at once and work is skipped.
  int it = 0;
  bool ok = true;
  for (int u = u0; u < U; ++u) {
    const long long iu0 = p.indptr[u], iu1 = p.indptr[u + 1];
    if (iu0 >= g1) break;
    const long long a = max(g0, iu0), b = min(g1, iu1);
    if (a >= b) continue;
    const int bb = u / p.Hkv, hkv = u % p.Hkv;
    named_bar_sync(1, nct);
    // q of the G query heads of this kv head, as fp32 and as 16-bit
    for (int i = tid; i < G * kHeadDim; i += nct) {
      const int h = i / kHeadDim, d = i % kHeadDim;
      const long long qi = ((long long)bb * p.Hq + (long long)hkv * G + h) * kHeadDim + d;
      const uint16_t raw = reinterpret_cast<const uint16_t*>(p.q)[qi];
      const float qf = p.q_bf16 ? __bfloat162float(__ushort_as_bfloat16(raw))
                                : __half2float(__ushort_as_half(raw));
      sm.q32[h][d] = qf;
      if constexpr (DENSE)
        sm.q16[h][d] = p.q_bf16 ? raw : __bfloat16_as_ushort(__float2bfloat16_rn(qf));
      else
        sm.q16[h][d] = p.q_bf16 ? __half_as_ushort(__float2half_rn(qf)) : raw;
      sm.O[h][d] = 0.0f;
    }
    named_bar_sync(1, nct);
    if constexpr (!DENSE) {
      for (int i = tid; i < 64 * kPairs; i += nct) {
        const int cc = i >> 6, pr = i & 63;
        const float cs = p.cos6[cc], sn = p.sin6[cc];
        uint16_t v[G];
#pragma unroll
        for (int h = 0; h < G; ++h)
          v[h] = __half_as_ushort(
              __float2half_rn(fmaf(sm.q32[h][2 * pr], cs, sm.q32[h][2 * pr + 1] * sn)));
        uint16_t* dst = sm.lut1 + i * G;
#pragma unroll
        for (int h = 0; h < G; ++h) dst[h] = v[h];
      }
      for (int i = tid; i < 16 * kPairs; i += nct) {
        const int cc = i >> 6, pr = i & 63;
        const float cs = p.cos4[cc], sn = p.sin4[cc];
        uint16_t* dst = sm.lut2 + i * G;
#pragma unroll
        for (int h = 0; h < G; ++h)
          dst[h] = __half_as_ushort(
              __float2half_rn(fmaf(sm.q32[h][2 * pr], cs, sm.q32[h][2 * pr + 1] * sn)));
      }
      named_bar_sync(1, nct);
    }
    WarpState st;
    st.m = -INFINITY;
    st.l = 0.0f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) st.acc[mt][e] = 0.0f;

    const long long nitems = (b - a + ipp - 1) / ipp;
    const int kpage = (8 * warp) >> p.log2P;
    const int row0 = (8 * warp) & (p.P - 1);
    for (long long i = 0; i < nitems; ++i, ++it) {
      const int s = it % kNSlot;
      if (ok && !mbar_wait_bounded(smem_u32(&sm.full[s]), (uint32_t)((it / kNSlot) & 1),
                                   &sm.abort_flag)) {
        ok = false;
        if (lane == 0) {
          report(p.err, SKV_ERR_TIMEOUT);
          sm.abort_flag = 1;
        }
      }
      if (ok && kpage < (int)sm.item_np[s]) {
        const uint32_t off = sm.item_off[s][kpage];
        if (off != kInvalidOff)
          process_rows<G, DENSE>(p, sm, ring + off, (sm.item_tier[s] >> (8 * kpage)) & 0xFFu,
                                 row0, st, lane);
      }
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(smem_u32(&sm.empty[s]));
    }

    // ---- combine the warps' states into this chunk's partial for unit u
    float l = st.l;
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 4);
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 8);
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 16);
    if (lane < G) {
      sm.ml[warp][lane][0] = st.m;
      sm.ml[warp][lane][1] = l;
    }
    named_bar_sync(1, nct);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int n = 2 * t4 + j;
      if (n < G) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kNCW; ++w) M = fmaxf(M, sm.ml[w][n][0]);
        const float mw = sm.ml[warp][n][0];
        const float sc = (mw == -INFINITY) ? 0.0f : exp2f(mw - M);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          atomicAdd(&sm.O[n][16 * mt + gq], st.acc[mt][j] * sc);
          atomicAdd(&sm.O[n][16 * mt + gq + 8], st.acc[mt][2 + j] * sc);
        }
      }
    }
    named_bar_sync(1, nct);
    float* part = p.part + (long long)(c + u) * G * kPartStride;
    for (int i = tid; i < G * kHeadDim; i += nct) {
      const int n = i / kHeadDim, d = i % kHeadDim;
      part[n * kPartStride + 4 + d] = sm.O[n][d];
      if (d == 0) {
        float M = -INFINITY;
        for (int w = 0; w < kNCW; ++w) M = fmaxf(M, sm.ml[w][n][0]);
        float L = 0.0f;
        if (M != -INFINITY)
          for (int w = 0; w < kNCW; ++w) {
            const float mw = sm.ml[w][n][0];
            if (mw != -INFINITY) L += sm.ml[w][n][1] * exp2f(mw - M);
          }
        part[n * kPartStride + 0] = M;
        part[n * kPartStride + 1] = L;
      }
    }
  }
}

// Merge the partials of every (unit, query head): one warp each.
template <int G>
__global__ void merge_kernel(const __grid_constant__ DecodeParams p) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int U = p.B * p.Hkv;
  if (wid >= U * G) return;
  const int u = wid / G, n = wid % G;
  const int bb = u / p.Hkv, hkv = u % p.Hkv;
  const long long N = p.indptr[U];
  const long long a = p.indptr[u], b = p.indptr[u + 1];
  const long long oi = ((long long)bb * p.Hq + (long long)hkv * G + n);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float M = -INFINITY, L = 0.0f;
  if (b > a && N > 0) {
    const long long S = p.S;
    const int c0 = (int)(((a + 1) * S - 1) / N);
    const int c1 = (int)((b * S - 1) / N);
    for (int c = c0; c <= c1; ++c) {
      if (chunk_begin(c, N, p.S) == chunk_begin(c + 1, N, p.S)) continue;
      const float m = p.part[(long long)(c + u) * G * kPartStride + n * kPartStride];
      M = fmaxf(M, m);
    }
    if (M != -INFINITY) {
      for (int c = c0; c <= c1; ++c) {
        if (chunk_begin(c, N, p.S) == chunk_begin(c + 1, N, p.S)) continue;
        const float* pp = p.part + (long long)(c + u) * G * kPartStride + n * kPartStride;
        const float m = pp[0];
        if (m == -INFINITY) continue;
        const float sc = exp2f(m - M);
        L += pp[1] * sc;
        const float4 o = *reinterpret_cast<const float4*>(pp + 4 + 4 * lane);
        acc.x += o.x * sc;
        acc.y += o.y * sc;
        acc.z += o.z * sc;
        acc.w += o.w * sc;
      }
    }
  }
  float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
  float lse = -INFINITY;
  if (L > 0.0f) {
    const float inv = 1.0f / L;
    res = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    lse = (M + log2f(L)) * 0.69314718055994530942f;
  }
  *reinterpret_cast<float4*>(p.out + oi * kHeadDim + 4 * lane) = res;
  if (p.lse && lane == 0) p.lse[oi] = lse;
}

template <int G, bool DENSE>
size_t decode_smem_fixed() {
  return ((sizeof(DecodeSmem<G, DENSE>) + 127) / 128) * 128;
}

template <int G, bool DENSE>
cudaError_t launch_decode_g(const DecodeParams& p, int ring_bytes, cudaStream_t stream,
                            cudaEvent_t between) {
  const size_t smem = decode_smem_fixed<G, DENSE>() + ring_bytes;
  // The shared-memory opt-in is set once per device and size (outside any
  // stream capture: the first call on a device is expected to be eager).
  static size_t configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || configured[dev] < smem) {
    e = cudaFuncSetAttribute(decode_kernel<G, DENSE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = smem;
  }
  decode_kernel<G, DENSE><<<p.S, kDecodeThreads, smem, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (between) {
    // an external record node when the stream is being captured into a graph
    e = cudaEventRecordWithFlags(between, stream, cudaEventRecordExternal);
    if (e != cudaSuccess) return e;
  }
  const int warps = p.B * p.Hkv * G;
  const int threads = 256;
  merge_kernel<G><<<(warps * 32 + threads - 1) / threads, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

size_t decode_fixed_smem(int G, bool dense) {
  if (dense) {
    switch (G) {
      case 1: return decode_smem_fixed<1, true>();
      case 2: return decode_smem_fixed<2, true>();
      default: return decode_smem_fixed<4, true>();
    }
  }
  switch (G) {
    case 1: return decode_smem_fixed<1, false>();
    case 2: return decode_smem_fixed<2, false>();
    default: return decode_smem_fixed<4, false>();
  }
}

cudaError_t launch_decode(const DecodeParams& p, int G, bool dense, cudaStream_t stream,
                          cudaEvent_t between) {
  if (dense) {
    switch (G) {
      case 1: return launch_decode_g<1, true>(p, p.ring_bytes, stream, between);
      case 2: return launch_decode_g<2, true>(p, p.ring_bytes, stream, between);
      case 4: return launch_decode_g<4, true>(p, p.ring_bytes, stream, between);
    }
  } else {
    switch (G) {
      case 1: return launch_decode_g<1, false>(p, p.ring_bytes, stream, between);
      case 2: return launch_decode_g<2, false>(p, p.ring_bytes, stream, between);
      case 4: return launch_decode_g<4, false>(p, p.ring_bytes, stream, between);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace skv
