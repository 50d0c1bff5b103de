// decode.cu -- ADA paged decode (SPHERICAL KV technical summary 2.1: logits
// computed directly from the radius and angle codes, no dense key
// materialised; 2.2: tier-homogeneous pages read in one header-guided pass)
// and the dense bf16 paged-decode baseline built on the same skeleton.
//
// Work split ("split-K over pages"): unit = (seq, kv head).  With at least
// 8 runs per unit each unit gets its own runs, in proportion to its
// streamed bytes, cut by bytes inside the unit; otherwise the CSR page list
// of all units (N pages) is cut into S runs of about equal streamed bytes
// (T0 pages cost 2.6x a T1 page).  CTA c streams run c and produces one
// partial (m, l, o) per unit it touches.  A unit covered by a single run
// is finished in place; otherwise the partial goes to slot c + u of the
// workspace and decode_merge_kernel, launched as a programmatic dependent
// of this grid, merges them (log-sum-exp); no CTA waits for another.
//
// CTA = kCG groups of 4 consumer warps + 1 planner warp + kIss issuer
// warps around one byte ring in shared memory.  The CTA's run is cut into
// "items" of 64 tokens (64/P pages, never crossing a unit).  The planner
// decodes page ids lane-parallel (a window of 64 pages at a time), places
// each item in the ring, writes its descriptors and signals it ready;
// issuer k copies the items i = k (mod kIss) with 1-D bulk asynchronous
// copies (no multicast), whole pages with their headers; consumer group g
// takes the items i = g (mod kCG), warp w of the group rows
// [64 w / kGW, 64 (w + 1) / kGW) of each, 16 rows per pass.  Slots carry
// ready (planner -> issuer), full (copies -> consumers) and empty
// (consumers -> planner) mbarriers.  The bulk-copy issue holds its thread
// for hundreds of cycles under load, so placement is kept off the issuing
// threads and several issuers run at once; one shared ring keeps several
// of even the largest (dense 64-token) items in flight.
//
// Consumer lane map: lane = 4 t + g, t = token of an 8-row group, g = dim
// group; each lane carries rows t and t + 8.  Logits of 16 rows: mma.sync
// m16n8k16 with A = the rows' keys and B = the G query heads (fp32
// accumulation): T0 / dense rows enter as they are stored (fp16 / bf16);
// T1 / T2 rows are rebuilt from their codes by gathers from a constant
// shared table of (share + 1) (cos, sin) per code in fp16 (one 4-byte,
// conflict-free gather per row and pair).  Lane (t, g) ends with the
// logits of head g of rows t and t + 8.  P.V: mma.sync m16n8k16, A = V^T
// fragments read straight from the page (pages store V in fragment order),
// B = P of the 16 rows x 8 heads (zero-padded beyond G), fp32 accumulation.
#include <algorithm>
#include <cstddef>

#include "common.cuh"
#include "kernels.h"

namespace skv {

#ifndef SKV_DECODE_ISSUERS
#define SKV_DECODE_ISSUERS 2
#endif
#ifndef SKV_DECODE_GROUPS
#define SKV_DECODE_GROUPS 3
#endif
constexpr int kGW = 4;                        // consumer warps per group
constexpr int kCG = SKV_DECODE_GROUPS;        // consumer groups
constexpr int kNCW = kCG * kGW;               // consumer warps per CTA
constexpr int kIss = SKV_DECODE_ISSUERS;      // issuer warps
constexpr int kPlannerWarp = kNCW;
constexpr int kDecodeThreads = (kNCW + 1 + kIss) * 32;
constexpr int kItemRows = 64;                 // tokens per item
constexpr int kRowsPerWarp = kItemRows / kGW;  // rows of an item per consumer warp
constexpr int kPasses = kRowsPerWarp / 16;
constexpr int kNSlot = 16;                    // items in flight, at most
constexpr int kMaxIPP = kItemRows / 16;       // pages per item (P >= 16)
constexpr int kMergeBatch = 20;               // merge: runs whose loads are issued together
constexpr int kTouchedUnits = 16;             // units whose segment costs a CTA keeps
constexpr int kStashRow = kHeadDim + 4;       // combine stash: floats per (warp, head) row
// Unit-aligned split: the last ~1/kDynDen of a unit's pages (whole chunks of
// kChunkItems items) are not cut into runs but handed out one chunk at a
// time, through a per-unit counter, to the unit's runs as they finish their
// static part; CTAs that stream faster take more of them.
#ifndef SKV_DYN_DEN
#define SKV_DYN_DEN 8
#endif
#ifndef SKV_CHUNK_ITEMS
#define SKV_CHUNK_ITEMS 8
#endif
constexpr int kDynDen = SKV_DYN_DEN;
constexpr int kChunkItems = SKV_CHUNK_ITEMS;
static_assert(kCG >= 1 && kCG <= 4, "consumer groups: 1..4");
static_assert(kIss >= 1 && kIss <= 4, "issuers: 1..4");
static_assert(kPasses >= 1 && kGW * kRowsPerWarp == kItemRows, "warp row split");

// Item descriptor (16 B, written by the producer before it arms the slot's
// full barrier): x = shared address of the item, y = meta, z/w = byte
// offsets of pages 1..3 from the item start (16 bits each).
// meta: bits 0-2 page count, bits 4 + 2k tier of page k, bit 12 + k page k
// unusable (bad id: nothing copied for it).
constexpr int kMetaTierShift = 4;
constexpr int kMetaBadShift = 12;
constexpr uint32_t kMetaUnitEnd = 1u << 20;  // a unit-end marker (desc.z: the next unit's first item)

// Shared-memory plan: [ring][TBL1][TBL2][fixed block] (ADA) or
// [ring][fixed block] (dense).  TBL1 / TBL2 are the reconstruction tables
// of the T1 / T2 codes (see build_tables): entry e at table + 128 e holds
// 32 copies of its 4 bytes, copy L read by lane L, so that a warp's
// gathers of any entries are one conflict-free wavefront.  TBL2 starts on
// an 8 KB boundary (its gather address is a LOP3 of the code bits and the
// lane's base); TBL1 sits right below it and the ring below TBL1.
constexpr uint32_t kTblEnt = 128;          // bytes per entry: 32 copies x 4 B
constexpr uint32_t kTbl1 = 256 * kTblEnt;   // T1: entry = code byte (angle6 << 2) | share2
constexpr uint32_t kTbl2 = 64 * kTblEnt;    // T2: entry = angle4 | share2 << 4

struct PageCopy {  // one page of a ready item, for its issuer
  uint32_t src_lo, src_hi, bytes, dst;
};

template <int G, bool DENSE>
struct __align__(16) DecodeSmem {
  unsigned long long full[kNSlot];
  unsigned long long empty[kNSlot];
  unsigned long long ready[kNSlot];
  uint4 desc[kNSlot];                  // consumers' view of an item
  PageCopy copy[kNSlot][kMaxIPP];      // issuers' view of an item
  uint32_t copy_bytes[kNSlot];         // bytes of the item (0xFFFFFFFF: no more items)
  uint32_t dpage[kNSlot];              // the item's first page (index into the page list)
  unsigned long long vstart[64];       // planner: virtual ring start of item j at j % 64
  unsigned long long scan[kDecodeThreads / 32];
  unsigned long long ucost[3 * kTouchedUnits + 1];  // cost before segments 3 unit0 ..
  unsigned long long ctot;             // total cost of the page list
  unsigned long long cunit[4];         // merge: cost before each segment of a unit, and its end
  long long useg[4];                   // merge: the unit's tier segment starts
  long long run[2];                    // this CTA's pages [run[0], run[1])
  long long dyn_m;                     // unit-aligned: first page of the unit's dynamic part
  int dyn_chunks, dyn_cp;              // its chunks and pages per chunk (0: no dynamic part)
  int dyn_first;                       // this run is its unit's first (resets the counter)
  int unit0, unit1;                    // the units of pages run[0] and run[1] - 1
  int abort_flag;
  int dyn_go;                          // consumers passed the wait for the previous grids
  int pad_[1];
  __align__(16) float ml[kNCW][4][2];
  float wsc[kNCW][4];                   // combine: each warp's scale per head
  float MH[4], LH[4];                   // combine: this CTA's (M, L) per head
  int c01[2];                           // the current unit's runs c0 .. c1
  __align__(16) float O[4][kHeadDim];
  __align__(16) float q32[4][kHeadDim];   // read with 16-byte shared loads
};
constexpr uint32_t kEndOfRun = 0xFFFFFFFFu;
using DecodeSmemG4 = DecodeSmem<4, false>;
static_assert(offsetof(DecodeSmemG4, q32) % 16 == 0, "q32 must be 16-byte aligned");
static_assert(offsetof(DecodeSmemG4, desc) % 16 == 0, "desc must be 16-byte aligned");

// Shared addresses of the ring, TBL1 (TBL2 follows it) and the fixed block
// for a dynamic shared window [base, limit).  False when the ring would be
// smaller than min_ring bytes.
template <int G, bool DENSE>
__host__ __device__ __forceinline__ bool smem_layout(uint32_t base, uint32_t limit,
                                                     uint32_t fixed_bytes, uint32_t min_ring,
                                                     uint32_t& ring_lo, uint32_t& ring_sz,
                                                     uint32_t& tbl1, uint32_t& fixed_at) {
  ring_lo = (base + 127) / 128 * 128;
  tbl1 = 0;
  if (limit < ring_lo + fixed_bytes + 128) return false;
  fixed_at = (limit - fixed_bytes) / 128 * 128;
  uint32_t ring_hi = fixed_at;
  if constexpr (!DENSE) {
    if (fixed_at < ring_lo + kTbl1 + kTbl2) return false;
    const uint32_t tbl2 = (fixed_at - kTbl2) / kTbl2 * kTbl2;
    if (tbl2 < ring_lo + kTbl1) return false;
    tbl1 = tbl2 - kTbl1;
    ring_hi = tbl1;
  }
  ring_sz = (ring_hi - ring_lo) / 128 * 128;
  return ring_sz >= min_ring;
}

// ---------------------------------------------------------------- the split
// The page list is cut into S runs of about equal streamed bytes (one per
// CTA).  Segment k = 3 u + t holds the tier-t pages of unit u (all pages
// count as tier 0 when no per-tier offsets are given); a page costs its
// tier's payload bytes.  With C(g) the cost of the pages before page g and
// C the total, page g belongs to run floor(C(g) S / C); run c starts at the
// first page g with C(g) S >= c C.  Every CTA scans the segment costs
// itself and keeps the prefix at the segments of the units it touches,
// which its merges need.
struct SplitInfo {
  const int32_t* indptr;
  const int32_t* tier_indptr;
  int U;
  int w[3];
  __device__ __forceinline__ long long seg_start(int k) const {
    if (tier_indptr) return tier_indptr[k];
    const int u = k / 3;
    return (k - 3 * u) == 0 ? indptr[u] : indptr[u + 1];
  }
  __device__ __forceinline__ unsigned long long weight(int k) const {
    const int t = k % 3;  // selects, not an indexed load: w stays in registers
    return (unsigned long long)(t == 0 ? w[0] : (t == 1 ? w[1] : w[2]));
  }
};

// floor(a / b) for b > 0.  Below 2^52 the quotient comes from one IEEE
// double division (a and b convert exactly; the rounded quotient is off by
// at most one) and is corrected with exact integer products, which keeps
// the 64-bit integer division sequence off the start-up path.
__device__ __forceinline__ unsigned long long udiv64(unsigned long long a, unsigned long long b) {
  if (a < (1ull << 52) && b < (1ull << 52)) {
    unsigned long long q = (unsigned long long)((double)a / (double)b);
    if (q * b > a)
      --q;
    else if ((q + 1) * b <= a)
      ++q;
    return q;
  }
  return a / b;
}

// First page of the run that starts at cost target T (= run index x total)
// among one unit's pages: seg[0..3] are the unit's tier segment starts,
// cseg[0..3] the costs before them; clamped to [seg[0], seg[3]].
__device__ __forceinline__ long long run_begin_in_unit(const SplitInfo& si,
                                                       const long long* seg,
                                                       const unsigned long long* cseg,
                                                       unsigned long long T,
                                                       unsigned long long S) {
  // unrolled with a result variable (constant indexes keep seg / cseg in
  // registers)
  long long res = seg[3];
  bool found = false;
#pragma unroll
  for (int t = 0; t < 3; ++t) {
    const unsigned long long lo = cseg[t] * S, hi = cseg[t + 1] * S;
    if (!found && T <= lo) {
      res = seg[t];
      found = true;
    } else if (!found && T <= hi) {
      const unsigned long long ws = si.weight(t) * S;
      res = seg[t] + (long long)udiv64(T - lo + ws - 1, ws);
      found = true;
    }
  }
  return res;
}

// Unit-aligned split (used when there are at most as many units as runs):
// unit u gets the runs [B(u), B(u + 1)), B(u) = u + round(P(u) (S - U) / C)
// with P(u) the cost before unit u and C the total -- at least one run per
// unit, the other S - U in proportion to cost -- and cuts them by cost
// within the unit.  No run crosses a unit, so no CTA pays a second unit's
// set-up, combine and merge for a sliver of pages.
#ifndef SKV_ALIGN_MIN_RUNS
#define SKV_ALIGN_MIN_RUNS 8
#endif
// The split is unit-aligned when every unit can have at least this many runs:
// rounding a unit's run count costs up to 1/n of its time, which beats the
// extra set-up and merge of runs that cross units only for n of about 8 and
// more (Llama-layer shapes with 2-3 runs per unit ran 11% faster on the
// global split).
constexpr int kAlignMinRuns = SKV_ALIGN_MIN_RUNS;
__host__ __device__ __forceinline__ bool unit_aligned_split(long long U, long long S) {
  return U * kAlignMinRuns <= S;
}

__device__ __forceinline__ int unit_first_run(int u, unsigned long long Pu, unsigned long long C,
                                              int S, int U) {
  if (C == 0) return u;
  return u + (int)udiv64(2ull * Pu * (unsigned long long)(S - U) + C, 2ull * C);
}

// This CTA's run [sm.run[0], sm.run[1]) (block-wide; contains barriers),
// its first and last unit, the total cost, and the cost before every
// segment of the units it touches (when they are at most kTouchedUnits).
template <class Smem>
__device__ __forceinline__ void find_run(const SplitInfo& si, int c, int S, Smem& sm, int tid,
                                      const uint32_t* ids, int ipp, bool dynamic) {
  constexpr int nt = kDecodeThreads;
  const int nseg = 3 * si.U;
  const int per = (nseg + nt - 1) / nt;
  const int k0 = min(nseg, tid * per), k1 = min(nseg, k0 + per);
  // the segment starts this thread needs in both passes (k0 .. k0 + 3, which
  // covers a unit's four when k0 starts one), loaded together: one memory
  // round trip on the start-up path
  long long pre[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) pre[t] = (k0 < k1 && k0 + t <= nseg) ? si.seg_start(k0 + t) : 0;
  unsigned long long loc = 0;
  if (per == 1) {
    if (k0 < k1) loc = (unsigned long long)(pre[1] - pre[0]) * si.weight(k0);
  } else {
    for (int k = k0; k < k1; ++k)
      loc += (unsigned long long)(si.seg_start(k + 1) - si.seg_start(k)) * si.weight(k);
  }
  if (k1 == nseg && k0 < k1) {
    // the page count is known: CTA c brings slice c of the page-id array into
    // L2, so that every planner's first id loads (after the split) hit L2
    const long long lines = (si.seg_start(nseg) * 4 + 127) / 128;
    const long long l0 = lines * c / S, l1 = lines * (c + 1) / S;
    for (long long l = l0; l < l1; ++l)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const uint8_t*>(ids) + 128 * l));
  }
  const int lane = tid & 31, w = tid >> 5;
  unsigned long long x = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm.scan[w] = x;
  if (tid == 0) {
    sm.run[0] = 0;  // the run boundaries that no segment claims (T = 0)
    sm.run[1] = 0;
    sm.unit0 = 0;
    sm.unit1 = -1;
    sm.dyn_chunks = 0;
    sm.dyn_cp = 0;
    sm.dyn_m = 0;
    sm.dyn_first = 0;
  }
  __syncthreads();
  unsigned long long before = x - loc, tot = 0;
#pragma unroll
  for (int i = 0; i < nt / 32; ++i) {
    if (i < w) before += sm.scan[i];
    tot += sm.scan[i];
  }
  const unsigned long long Su = (unsigned long long)S;
  const bool aligned = unit_aligned_split(si.U, S);
  unsigned long long cc = before;
  if (aligned) {
    // the thread holding the first segment of unit u knows P(u) and the
    // unit's segments: if c is among u's runs [B(u), B(u + 1)) it writes the
    // whole split of this CTA (run j of n: its share of the unit's cost)
    for (int k = k0; k < k1; ++k) {
      if (k % 3 == 0) {
        const int u = k / 3;
        long long seg[4];
        unsigned long long cr[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) seg[t] = (k == k0) ? pre[t] : si.seg_start(k + t);
        cr[0] = 0;
#pragma unroll
        for (int t = 0; t < 3; ++t) cr[t + 1] = cr[t] + (unsigned long long)(seg[t + 1] - seg[t]) * si.weight(t);
        const int B0 = unit_first_run(u, cc, tot, S, si.U);
        const int B1 = unit_first_run(u + 1, cc + cr[3], tot, S, si.U);
        if (B0 <= c && c < B1) {
          const int n = B1 - B0, j = c - B0;
          sm.unit0 = u;
          sm.unit1 = u;
#pragma unroll
          for (int t = 0; t < 4; ++t) sm.ucost[t] = cc + cr[t];
          // the dynamic part: whole chunks at the end of the unit, about
          // 1/kDynDen of its pages (none for a unit with a single run); the
          // static part [seg[0], M) is cut into the n runs by cost
          const long long cp = (long long)kChunkItems * ipp;
          const long long nch =
              (dynamic && n >= 2) ? (long long)udiv64((unsigned long long)(seg[3] - seg[0]), kDynDen * cp) : 0;
          const long long M = seg[3] - nch * cp;
          long long sg[4];
          unsigned long long cs[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) sg[t] = min(seg[t], M);
          cs[0] = 0;
#pragma unroll
          for (int t = 0; t < 3; ++t) cs[t + 1] = cs[t] + (unsigned long long)(sg[t + 1] - sg[t]) * si.weight(t);
          sm.run[0] = run_begin_in_unit(si, sg, cs, (unsigned long long)j * cs[3], (unsigned long long)n);
          sm.run[1] = run_begin_in_unit(si, sg, cs, (unsigned long long)(j + 1) * cs[3], (unsigned long long)n);
          sm.dyn_m = M;
          sm.dyn_chunks = (int)nch;
          sm.dyn_cp = (int)cp;
          sm.dyn_first = j == 0;
        }
      }
      cc += (unsigned long long)(si.seg_start(k + 1) - si.seg_start(k)) * si.weight(k);
    }
    if (tid == 0) sm.ctot = tot;
    __syncthreads();
    return;
  } else {
    const unsigned long long T0 = (unsigned long long)c * tot, T1 = (unsigned long long)(c + 1) * tot;
    for (int k = k0; k < k1; ++k) {
      const long long a = si.seg_start(k), b = si.seg_start(k + 1);
      const unsigned long long ws = si.weight(k) * Su;
      const unsigned long long lo = cc * Su, hi = lo + (unsigned long long)(b - a) * ws;
      if (lo < T0 && T0 <= hi) sm.run[0] = a + (long long)udiv64(T0 - lo + ws - 1, ws);
      if (lo < T1 && T1 <= hi) sm.run[1] = a + (long long)udiv64(T1 - lo + ws - 1, ws);
      cc += (unsigned long long)(b - a) * si.weight(k);
    }
  }
  if (tid == 0) sm.ctot = tot;
  __syncthreads();
  {
    // the units of the run's first and last page (their segments hold them)
    const long long g0 = sm.run[0], g1 = sm.run[1];
    for (int k = k0; k < k1; ++k) {
      const long long a = si.seg_start(k), b = si.seg_start(k + 1);
      if (a <= g0 && g0 < b) sm.unit0 = k / 3;
      if (a < g1 && g1 <= b) sm.unit1 = k / 3;
    }
  }
  __syncthreads();
  const int ua = sm.unit0, ub = sm.unit1;
  if (ub >= ua && ub - ua < kTouchedUnits) {
    cc = before;
    for (int k = k0; k < k1; ++k) {
      if (k >= 3 * ua && k <= 3 * ub + 3) sm.ucost[k - 3 * ua] = cc;
      cc += (unsigned long long)(si.seg_start(k + 1) - si.seg_start(k)) * si.weight(k);
    }
    // the cost after the last segment (the end of the page list)
    if (k1 == nseg && k0 < k1 && nseg <= 3 * ub + 3) sm.ucost[nseg - 3 * ua] = cc;
  }
  __syncthreads();
}

// A 32-bit tag of this grid launch (the low half of the temporal grid
// identifier, which differs between launches in a context).
__device__ __forceinline__ uint32_t launch_tag() {
  unsigned long long g;
  asm volatile("mov.u64 %0, %%gridid;" : "=l"(g));
  return (uint32_t)g;
}

__device__ __forceinline__ int ld_volatile(const int* p) {
  return *reinterpret_cast<const volatile int*>(p);
}

// ------------------------------------------------------ shared loads (PTX) --
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}

// ------------------------------------------------------ logits (mma.sync) --
// Logits of 16 rows are one m16n8k16 MMA chain: A = the rows' keys (16 rows
// x 16 dims per k-step), B = the query heads (16 dims x 8 columns), fp32
// accumulation.  Column n holds head (n / 2) % G for even n and zeros for
// odd n, so that C element c0 (row t, column 2 g) of lane (t, g) is the
// logit of head g % G and row t, c2 that of row t + 8: the layout the
// online softmax takes, with no reduction across lanes.
//
// The k index is a permutation of the dims fixed by what a lane reads of a
// row: lane (t, g) reads dims 32 i + 8 g + 0..7 (i = 0..3) of a T0 or dense
// row (chunk 4 i + g) and the codes of the same dims' pairs 16 i + 4 g + 0..3
// of a T1 / T2 row.  K-step 2 i + h takes, for lane (t, g), the dims
// 32 i + 8 g + 4 h + {0, 1} as k = 2 g, 2 g + 1 and + {2, 3} as k = 2 g + 8,
// 2 g + 9; B follows the same map.
struct QFrag {
  uint32_t b[16];   // B fragments, k-step s in b[2 s], b[2 s + 1]
  uint32_t lo[16];  // dense kernel with fp16 q: the low bf16 halves of q
  bool two;         // dense kernel: lo is in use
  float c0;         // logit scale (log2 domain) of fp16 / bf16 keys, this lane's head
  float c1;         // the same for codes (shares entered as code + 1 = 16 rho^)
};

__device__ __forceinline__ float pow2f(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// B fragments of this lane's column from the fp32 query rows q32[head][dim].
// ADA: keys are fp16, so q enters as fp16 scaled by a power of two per head
// (its largest element to [2^14, 2^15): bf16 and fp16 queries convert
// exactly), the scale being taken off in c0 / c1.  Dense: keys are bf16; a
// bf16 q enters as it is, an fp16 q as the sum of two bf16 halves (exact).
template <int G, bool DENSE>
__device__ __forceinline__ void make_qfrag(const float (*q32)[kHeadDim], float qk_scale_log2,
                                           bool q_bf16, int lane, QFrag& f) {
  const int gq = lane >> 2, t4 = lane & 3;
  const bool live = (gq & 1) == 0;
  const int hn = (gq >> 1) % G;
  float mx = 0.0f;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const float4 x = *reinterpret_cast<const float4*>(&q32[hn][32 * (s >> 1) + 8 * t4 + 4 * (s & 1)]);
    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
  }
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
  int e = 0;
  if (!DENSE && mx > 0.0f) e = min(126, 141 - (int)((__float_as_uint(mx) >> 23) & 0xFFu));
  const float sc = pow2f(e);
  f.two = DENSE && !q_bf16;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    float4 x = *reinterpret_cast<const float4*>(&q32[hn][32 * (s >> 1) + 8 * t4 + 4 * (s & 1)]);
    if (!live) x = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if constexpr (DENSE) {
      f.b[2 * s] = pack_bf16x2(x.x, x.y);
      f.b[2 * s + 1] = pack_bf16x2(x.z, x.w);
      const float hx = __uint_as_float(f.b[2 * s] << 16), hy = __uint_as_float(f.b[2 * s] & 0xFFFF0000u);
      const float hz = __uint_as_float(f.b[2 * s + 1] << 16),
                  hw = __uint_as_float(f.b[2 * s + 1] & 0xFFFF0000u);
      f.lo[2 * s] = pack_bf16x2(x.x - hx, x.y - hy);
      f.lo[2 * s + 1] = pack_bf16x2(x.z - hz, x.w - hw);
    } else {
      f.b[2 * s] = pack_f16x2(x.x * sc, x.y * sc);
      f.b[2 * s + 1] = pack_f16x2(x.z * sc, x.w * sc);
    }
  }
  // the lane's own head (column 2 t4) is the column of lane 8 t4
  const float inv = __shfl_sync(0xFFFFFFFFu, pow2f(-e), 8 * t4);
  f.c0 = qk_scale_log2 * inv;
  f.c1 = qk_scale_log2 * 0.0625f * inv;
}

// Reconstruction tables: T1 entry e = (a << 2) | s and T2 entry 256 + (a | s << 4)
// hold the pair (x, y) = (s + 1) (cos, sin)(2 pi a / 2^b) (16 times the
// key pair of unit radius: shares enter as code + 1) rounded to fp16
// (relative error <= 2^-11 per component; the logit of a row is the
// fp32-accumulated sum of exact fp16 x fp16 products).  The T2 entries
// follow T1's (TBL2 = TBL1 + 32 KB).  Eight threads fill one entry's 128
// bytes with 16-byte stores, so a warp writes 512 contiguous bytes.
// VAR bit 0: the T1 variant, code byte (angle5 << 3) | share3 with weight
// (s + 1) / 2; bit 1: the 2-bit share codes on the Lloyd-Max grid, weights
// 2 u_s = {766, 1614, 2498, 3662} / 1024 instead of s + 1 (share u_s / 8).
template <int VAR>
__device__ __forceinline__ float share2_weight(uint32_t s) {
  if constexpr ((VAR & 2) != 0)
    return s == 0 ? 766.0f / 1024 : (s == 1 ? 1614.0f / 1024 : (s == 2 ? 2498.0f / 1024 : 3662.0f / 1024));
  else
    return (float)(s + 1);
}

template <int VAR>
__device__ __forceinline__ void build_tables(const DecodeParams& p, uint8_t* tbl1p, int n_entries,
                                             int tid, int nthreads) {
  for (int i = tid; i < 8 * n_entries; i += nthreads) {
    const int e = i >> 3;
    float cs, sn, w;
    if ((VAR & 1) && e < 256) {
      cs = p.cos5[e >> 3];
      sn = p.sin5[e >> 3];
      w = 0.5f * (float)((e & 7) + 1);
    } else if (e < 256) {
      cs = p.cos6[e >> 2];
      sn = p.sin6[e >> 2];
      w = share2_weight<VAR>((uint32_t)e & 3u);
    } else {
      cs = p.cos4[(e - 256) & 15];
      sn = p.sin4[(e - 256) & 15];
      w = share2_weight<VAR>((uint32_t)(e - 256) >> 4);
    }
    const float x = w * cs, y = w * sn;
    const uint32_t h = pack_f16x2(x, y);
    reinterpret_cast<uint4*>(tbl1p)[i] = make_uint4(h, h, h, h);
  }
}

template <bool BF16>
__device__ __forceinline__ void mma_k16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (BF16)
    mma_16816k16_bf16(d, a0, a1, a2, a3, b0, b1);
  else
    mma_16816k16_f16(d, a0, a1, a2, a3, b0, b1);
}

// T0 (fp16 K) or dense (bf16 K) rows rA, rA + 8: lane (t, g) reads chunks
// c = 4 i + g (dims 8 c .. 8 c + 7), stored at chunk position c ^ 4 (row & 1).
// Two accumulators (even / odd k-steps) halve the MMA dependency chain.
template <bool BF16, bool TWO>
__device__ __forceinline__ void logits_k16(uint32_t pg, int rA, int g, const QFrag& f,
                                           float (&c)[4], float (&d)[4]) {
  const uint32_t ka = pg + kHdrBytes + rA * 256;
  const uint32_t kb = ka + 8 * 256;
  const uint32_t sw = 4u * (rA & 1);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t pos = (((uint32_t)(4 * i + g)) ^ sw) * 16;
    const uint4 xa = lds128(ka + pos), xb = lds128(kb + pos);
    mma_k16<BF16>(c, xa.x, xb.x, xa.y, xb.y, f.b[4 * i], f.b[4 * i + 1]);
    mma_k16<BF16>(d, xa.z, xb.z, xa.w, xb.w, f.b[4 * i + 2], f.b[4 * i + 3]);
    if constexpr (TWO) {
      mma_k16<BF16>(c, xa.x, xb.x, xa.y, xb.y, f.lo[4 * i], f.lo[4 * i + 1]);
      mma_k16<BF16>(d, xa.z, xb.z, xa.w, xb.w, f.lo[4 * i + 2], f.lo[4 * i + 3]);
    }
  }
}

// table address of code byte k of w (T1: entry = the byte)
__device__ __forceinline__ uint32_t t1_addr(uint32_t w, int k, uint32_t tb) {
  return tb + (__byte_perm(w, 0u, 0x4440u | (uint32_t)k) << 7);
}

// T1 rows rA, rA + 8: lane (t, g) reads code bytes [16 g, 16 g + 16) of
// each row; byte j holds pair 16 (j >> 2) + 4 g + (j & 3), so k-step s uses
// bytes 2 s (k = 2 g, 2 g + 1) and 2 s + 1 (k = 2 g + 8, 2 g + 9).  Even and
// odd k-steps go to separate accumulators (two MMA chains of four).
__device__ __forceinline__ void logits_t1(uint32_t pg, int P, int rA, int g, uint32_t tb,
                                          const QFrag& f, float (&c)[4], float (&d)[4]) {
  const uint32_t cd = pg + kHdrBytes + 2 * P;
  const uint4 ca = lds128(cd + rA * 64 + 16 * g);
  const uint4 cb = lds128(cd + (rA + 8) * 64 + 16 * g);
  const uint32_t wa[4] = {ca.x, ca.y, ca.z, ca.w};
  const uint32_t wb[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int i = s >> 1, k0 = 2 * (s & 1);
    const uint32_t ea0 = lds32(t1_addr(wa[i], k0, tb)), ea1 = lds32(t1_addr(wa[i], k0 + 1, tb));
    const uint32_t eb0 = lds32(t1_addr(wb[i], k0, tb)), eb1 = lds32(t1_addr(wb[i], k0 + 1, tb));
    if (s & 1)
      mma_k16<false>(d, ea0, eb0, ea1, eb1, f.b[2 * s], f.b[2 * s + 1]);
    else
      mma_k16<false>(c, ea0, eb0, ea1, eb1, f.b[2 * s], f.b[2 * s + 1]);
  }
}

// table address of T2 pair j: nibble j of the 64-bit nibble word (n0, n1),
// crumb j of the share word cw; entry angle | share << 4 (TBL2 is 8 KB
// aligned: the address is tb | entry << 7; j is a constant once unrolled)
__device__ __forceinline__ uint32_t t2_addr(uint32_t n0, uint32_t n1, uint32_t cw, int j,
                                            uint32_t tb) {
  const int sn = 4 * (j & 7) - 7, sc = 2 * j - 11;
  const uint32_t nw = j < 8 ? n0 : n1;
  const uint32_t xn = sn >= 0 ? (nw >> sn) : (nw << -sn);
  const uint32_t xc = sc >= 0 ? (cw >> sc) : (cw << -sc);
  return (xn & 0x780u) | (xc & 0x1800u) | tb;
}

// T2 rows rA, rA + 8: nibble j of bytes [8 g, 8 g + 8) holds the angle of
// pair 16 (j >> 2) + 4 g + (j & 3), crumb j of bytes [32 + 4 g, 36 + 4 g) its share.
__device__ __forceinline__ void logits_t2(uint32_t pg, int P, int rA, int g, uint32_t tb,
                                          const QFrag& f, float (&c)[4], float (&d)[4]) {
  const uint32_t cd = pg + kHdrBytes + 2 * P;
  const uint2 na = lds64(cd + rA * 48 + 8 * g);
  const uint2 nb = lds64(cd + (rA + 8) * 48 + 8 * g);
  const uint32_t ra = lds32(cd + rA * 48 + 32 + 4 * g);
  const uint32_t rb = lds32(cd + (rA + 8) * 48 + 32 + 4 * g);
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const uint32_t ea0 = lds32(t2_addr(na.x, na.y, ra, 2 * s, tb));
    const uint32_t ea1 = lds32(t2_addr(na.x, na.y, ra, 2 * s + 1, tb));
    const uint32_t eb0 = lds32(t2_addr(nb.x, nb.y, rb, 2 * s, tb));
    const uint32_t eb1 = lds32(t2_addr(nb.x, nb.y, rb, 2 * s + 1, tb));
    if (s & 1)
      mma_k16<false>(d, ea0, eb0, ea1, eb1, f.b[2 * s], f.b[2 * s + 1]);
    else
      mma_k16<false>(c, ea0, eb0, ea1, eb1, f.b[2 * s], f.b[2 * s + 1]);
  }
}

struct WarpState {
  float m;          // running max (log2 domain) of head g % G, or kNoMax
  float l;          // partial denominator of (token slot t, head g % G)
  float acc[8][4];  // O^T fragments: [m-tile][c0..c3]
  float ones[4];    // sum of the P.V B operand per head (int8 V bias, see softmax_pv)
};

// Start value of the running max: finite, so that exp2 of (-inf - m) is 0
// and never NaN; any real logit is far above it.
constexpr float kNoMax = -1.0e30f;
// The running max is raised (and the accumulators rescaled) only when a
// logit exceeds it by more than this (log2 units): weights then stay below
// 2^4 and most 16-row steps skip the rescale.
constexpr float kLazyMax = 4.0f;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Online softmax of 16 rows and P.V into the accumulators.
// lA / lB: log2-domain logits of rows t and t + 8 (head g % G) or -inf.
// VK: 0 int8 V (1 KB per 8-row group), 1 fp16 V, 2 bf16 V (2 KB per group).
// The online-softmax update of 16 rows: raises the running max when needed
// (rescaling the accumulators), adds the rows' weights to l and returns the
// P.V B fragments (k16 x n8: k = rows 2t4, 2t4+1 | 8+2t4, 9+2t4, n = head
// gq) of the weights times the rows' V scales, as fp16 (F16) or bf16.
template <int G, bool F16>
__device__ __forceinline__ void softmax_weights(float lA, float lB, float vsA, float vsB,
                                                WarpState& st, int lane, uint32_t& bf0,
                                                uint32_t& bf1) {
  const int gq = lane >> 2, t4 = lane & 3;
  if (__any_sync(0xFFFFFFFFu, fmaxf(lA, lB) > st.m + kLazyMax)) {
    float cm = fmaxf(lA, lB);
    cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 4));
    cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 8));
    cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 16));
    const float m_new = fmaxf(st.m, cm);
    const float alpha = ex2_approx(st.m - m_new);  // 0 when st.m is kNoMax
    st.l *= alpha;
    st.m = m_new;
    const int n0 = 2 * t4, n1 = 2 * t4 + 1;
    const float a0 = __shfl_sync(0xFFFFFFFFu, alpha, n0 < G ? n0 : 0);
    const float a1 = __shfl_sync(0xFFFFFFFFu, alpha, n1 < G ? n1 : 0);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      st.acc[mt][0] *= a0;
      st.acc[mt][1] *= a1;
      st.acc[mt][2] *= a0;
      st.acc[mt][3] *= a1;
    }
    st.ones[0] *= a0;
    st.ones[1] *= a1;
    st.ones[2] *= a0;
    st.ones[3] *= a1;
  }
  const float pA = ex2_approx(lA - st.m), pB = ex2_approx(lB - st.m);  // -inf -> 0
  st.l += pA + pB;
  const float ppA = pA * vsA, ppB = pB * vsB;
  const int src = 8 * t4 + (gq < G ? gq : 0);
  const float b0 = __shfl_sync(0xFFFFFFFFu, ppA, src);
  const float b1 = __shfl_sync(0xFFFFFFFFu, ppA, src + 4);
  const float b2 = __shfl_sync(0xFFFFFFFFu, ppB, src);
  const float b3 = __shfl_sync(0xFFFFFFFFu, ppB, src + 4);
  bf0 = F16 ? pack_f16x2(b0, b1) : pack_bf16x2(b0, b1);
  bf1 = F16 ? pack_f16x2(b2, b3) : pack_bf16x2(b2, b3);
}

// P.V of 16 int8 V rows already in registers (fragment words of the two
// 8-row blocks), v + 1152 as fp16, the bias taken off through the ones MMA.
__device__ __forceinline__ void pv_int8_regs(const uint32_t (&wa)[8], const uint32_t (&wb)[8],
                                             uint32_t bf0, uint32_t bf1, WarpState& st) {
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    uint32_t a0, a1, a2, a3;
    s8x4_to_f16x2x2_biased(wa[mt], a0, a1);
    s8x4_to_f16x2x2_biased(wb[mt], a2, a3);
    mma_16816k16_f16(st.acc[mt], a0, a1, a2, a3, bf0, bf1);
  }
  constexpr uint32_t kOnes = 0x3C003C00u;  // fp16 (1, 1)
  mma_16816k16_f16(st.ones, kOnes, kOnes, kOnes, kOnes, bf0, bf1);
}

template <int G, int VK>
__device__ __forceinline__ void softmax_pv(float lA, float lB, float vsA, float vsB, uint32_t va,
                                           uint32_t vb, WarpState& st, int lane) {
  const int gq = lane >> 2, t4 = lane & 3;
  // a lane's own rows decide whether the running max must rise; only then
  // is the max over the 16 rows (lanes of the same head) formed
  if (__any_sync(0xFFFFFFFFu, fmaxf(lA, lB) > st.m + kLazyMax)) {
    float cm = fmaxf(lA, lB);
    cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 4));
    cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 8));
    cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 16));
    const float m_new = fmaxf(st.m, cm);
    const float alpha = ex2_approx(st.m - m_new);  // 0 when st.m is kNoMax
    st.l *= alpha;
    st.m = m_new;
    const int n0 = 2 * t4, n1 = 2 * t4 + 1;
    const float a0 = __shfl_sync(0xFFFFFFFFu, alpha, n0 < G ? n0 : 0);
    const float a1 = __shfl_sync(0xFFFFFFFFu, alpha, n1 < G ? n1 : 0);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      st.acc[mt][0] *= a0;
      st.acc[mt][1] *= a1;
      st.acc[mt][2] *= a0;
      st.acc[mt][3] *= a1;
    }
    st.ones[0] *= a0;
    st.ones[1] *= a1;
    st.ones[2] *= a0;
    st.ones[3] *= a1;
  }
  const float pA = ex2_approx(lA - st.m), pB = ex2_approx(lB - st.m);  // -inf -> 0
  st.l += pA + pB;
  const float ppA = pA * vsA, ppB = pB * vsB;
  // B fragment (k16 x n8): k = rows 2t4, 2t4+1 | 8+2t4, 9+2t4, n = head gq
  const int src = 8 * t4 + (gq < G ? gq : 0);
  // columns n >= G (lanes gq >= G) carry copies of head 0: their outputs
  // are never read
  const float b0 = __shfl_sync(0xFFFFFFFFu, ppA, src);
  const float b1 = __shfl_sync(0xFFFFFFFFu, ppA, src + 4);
  const float b2 = __shfl_sync(0xFFFFFFFFu, ppB, src);
  const float b3 = __shfl_sync(0xFFFFFFFFu, ppB, src + 4);
  if constexpr (VK == 0) {
    // int8 V enters the MMA as the fp16 value v + 1152 (exact: 0x64XX with
    // XX = v + 128); one more MMA against an all-ones A tile accumulates the
    // B column sums, and 1152 times them is taken off when the warps'
    // states are combined
    const uint32_t bf0 = pack_f16x2(b0, b1), bf1 = pack_f16x2(b2, b3);
    const uint4 xa = lds128(va + lane * 16), ya = lds128(va + 512 + lane * 16);
    const uint4 xb = lds128(vb + lane * 16), yb = lds128(vb + 512 + lane * 16);
    const uint32_t wa[8] = {xa.x, xa.y, xa.z, xa.w, ya.x, ya.y, ya.z, ya.w};
    const uint32_t wb[8] = {xb.x, xb.y, xb.z, xb.w, yb.x, yb.y, yb.z, yb.w};
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t a0, a1, a2, a3;
      s8x4_to_f16x2x2_biased(wa[mt], a0, a1);
      s8x4_to_f16x2x2_biased(wb[mt], a2, a3);
      mma_16816k16_f16(st.acc[mt], a0, a1, a2, a3, bf0, bf1);
    }
    constexpr uint32_t kOnes = 0x3C003C00u;  // fp16 (1, 1)
    mma_16816k16_f16(st.ones, kOnes, kOnes, kOnes, kOnes, bf0, bf1);
  } else {
    const uint32_t bf0 = (VK == 1) ? pack_f16x2(b0, b1) : pack_bf16x2(b0, b1);
    const uint32_t bf1 = (VK == 1) ? pack_f16x2(b2, b3) : pack_bf16x2(b2, b3);
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
      const uint4 za = lds128(va + qq * 512 + lane * 16);
      const uint4 zb = lds128(vb + qq * 512 + lane * 16);
      if constexpr (VK == 1) {
        mma_16816k16_f16(st.acc[2 * qq], za.x, za.y, zb.x, zb.y, bf0, bf1);
        mma_16816k16_f16(st.acc[2 * qq + 1], za.z, za.w, zb.z, zb.w, bf0, bf1);
      } else {
        mma_16816k16_bf16(st.acc[2 * qq], za.x, za.y, zb.x, zb.y, bf0, bf1);
        mma_16816k16_bf16(st.acc[2 * qq + 1], za.z, za.w, zb.z, zb.w, bf0, bf1);
      }
    }
  }
}

// Lane (t, g) holds the log2-domain logits of head g for rows rA and rB;
// with capture on, heads g < G store them at lg[row * G + g] (the 8 rows of
// a half-step and their G heads are contiguous: one 32 G-byte segment).
template <int G>
__device__ __forceinline__ void capture_logits(float* lg, int rA, int rB, bool vA, bool vB,
                                               float lA, float lB, int g) {
  if (lg != nullptr && g < G) {
    if (vA) lg[rA * G + g] = lA;
    if (vB) lg[rB * G + g] = lB;
  }
}

// 16 rows [row0, row0 + 16) of one page at shared address pg; tb1 / tb2:
// this lane's copy in TBL1 / TBL2; lg: the page's logit rows, or NULL
// (CAP: the kernel variant that captures logits).  T0B: the fused T0 / bf16
// path, whose T0 pages hold bf16 K / V and take the dense kernel's logit and
// P.V steps, with bf16 fragments of q formed from q32 for the page.
template <int G, bool DENSE, bool CAP, bool T0B>
__device__ __forceinline__ void process_rows(const DecodeParams& p, uint32_t pg, uint32_t tier,
                                             int row0, const QFrag& qf, uint32_t tb1,
                                             uint32_t tb2, WarpState& st, int lane, float* lg,
                                             const float (*q32)[kHeadDim]) {
  const int t = lane >> 2, g = lane & 3;
  const int P = p.P;
  // header {u16 count, u8 tier, u8 magic}
  const uint32_t h0 = lds32(pg);
  const uint32_t cnt = h0 & 0xFFFFu;
  if ((h0 >> 16) != (tier | ((uint32_t)kPageMagic << 8)) || cnt > (uint32_t)P) {
    if (lane == 0) report(p.err, SKV_ERR_CORRUPT);
    return;
  }
  if ((uint32_t)row0 >= cnt) return;
  const int rA = row0 + t, rB = rA + 8;
  const bool vA = (uint32_t)rA < cnt, vB = (uint32_t)rB < cnt;
  float c[4] = {0.0f, 0.0f, 0.0f, 0.0f}, d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  const uint32_t vsec_dense = pg + kHdrBytes + 256 * P + (row0 >> 3) * 2048;
  if constexpr (DENSE) {
    if (qf.two)
      logits_k16<true, true>(pg, rA, g, qf, c, d);
    else
      logits_k16<true, false>(pg, rA, g, qf, c, d);
    const float a = c[0] + d[0], b = c[2] + d[2];
    softmax_pv<G, 2>(vA ? a * qf.c0 : -INFINITY, vB ? b * qf.c0 : -INFINITY, 1.0f, 1.0f,
                     vsec_dense, vsec_dense + 2048, st, lane);
  } else {
    if (T0B && tier == SKV_TIER_T0) {
      QFrag qb;
      make_qfrag<G, true>(q32, p.qk_scale_log2, p.q_bf16 != 0, lane, qb);
      if (qb.two)
        logits_k16<true, true>(pg, rA, g, qb, c, d);
      else
        logits_k16<true, false>(pg, rA, g, qb, c, d);
      const float lA = vA ? (c[0] + d[0]) * qb.c0 : -INFINITY;
      const float lB = vB ? (c[2] + d[2]) * qb.c0 : -INFINITY;
      if constexpr (CAP) capture_logits<G>(lg, rA, rB, vA, vB, lA, lB, g);
      softmax_pv<G, 2>(lA, lB, 1.0f, 1.0f, vsec_dense, vsec_dense + 2048, st, lane);
    } else if (tier == SKV_TIER_T0) {
      logits_k16<false, false>(pg, rA, g, qf, c, d);
      const float lA = vA ? (c[0] + d[0]) * qf.c0 : -INFINITY;
      const float lB = vB ? (c[2] + d[2]) * qf.c0 : -INFINITY;
      if constexpr (CAP) capture_logits<G>(lg, rA, rB, vA, vB, lA, lB, g);
      softmax_pv<G, 1>(lA, lB, 1.0f, 1.0f, vsec_dense, vsec_dense + 2048, st, lane);
    } else {
      const bool t1 = tier == SKV_TIER_T1;
      if (t1)
        logits_t1(pg, P, rA, g, tb1, qf, c, d);
      else
        logits_t2(pg, P, rA, g, tb2, qf, c, d);
      const float a = c[0] + d[0], b = c[2] + d[2];
      const int cb = t1 ? 64 : 48;
      const uint32_t rs = pg + kHdrBytes, ss = pg + kHdrBytes + (2 + cb) * P;
      const float rtA = __half2float(__ushort_as_half((unsigned short)lds16(rs + 2 * rA)));
      const float rtB = __half2float(__ushort_as_half((unsigned short)lds16(rs + 2 * rB)));
      const float vsA = __half2float(__ushort_as_half((unsigned short)lds16(ss + 2 * rA)));
      const float vsB = __half2float(__ushort_as_half((unsigned short)lds16(ss + 2 * rB)));
      const uint32_t vsec = pg + kHdrBytes + (2 + cb + 2) * P + (row0 >> 3) * 1024;
      const float lA = vA ? a * (rtA * qf.c1) : -INFINITY;
      const float lB = vB ? b * (rtB * qf.c1) : -INFINITY;
      if constexpr (CAP) capture_logits<G>(lg, rA, rB, vA, vB, lA, lB, g);
      softmax_pv<G, 0>(lA, lB, vA ? vsA : 0.0f, vB ? vsB : 0.0f, vsec, vsec + 1024, st, lane);
    }
  }
}

// The ring data a lane needs for 16 T1 / T2 rows of one page: the page's
// header word, the lane's code words of rows rA and rA + 8, their radii and V
// scales (fp16 bits, row A low), and its int8 V fragment words.  Loaded all
// at once, so that the item's ring space can be released before the rows
// are computed (the consumers then hold only registers, not ring bytes).
struct CodeRows {
  uint32_t hdr;
  uint32_t ca[4], cb[4];  // T1: the 16 code bytes of each row; T2: nibbles (2) + crumbs (1)
  uint32_t rs, vs;
  uint32_t va[8], vb[8];
};

__device__ __forceinline__ void load_code_rows(uint32_t pg, int P, bool t1, int row0, int lane,
                                               CodeRows& r) {
  const int t = lane >> 2, g = lane & 3;
  const int rA = row0 + t, rB = rA + 8;
  r.hdr = lds32(pg);
  const uint32_t cd = pg + kHdrBytes + 2 * P;
  int cb;
  if (t1) {
    const uint4 a = lds128(cd + rA * 64 + 16 * g), b = lds128(cd + rB * 64 + 16 * g);
    r.ca[0] = a.x; r.ca[1] = a.y; r.ca[2] = a.z; r.ca[3] = a.w;
    r.cb[0] = b.x; r.cb[1] = b.y; r.cb[2] = b.z; r.cb[3] = b.w;
    cb = 64;
  } else {
    const uint2 na = lds64(cd + rA * 48 + 8 * g), nb = lds64(cd + rB * 48 + 8 * g);
    r.ca[0] = na.x; r.ca[1] = na.y; r.ca[2] = lds32(cd + rA * 48 + 32 + 4 * g); r.ca[3] = 0u;
    r.cb[0] = nb.x; r.cb[1] = nb.y; r.cb[2] = lds32(cd + rB * 48 + 32 + 4 * g); r.cb[3] = 0u;
    cb = 48;
  }
  const uint32_t rsec = pg + kHdrBytes, ssec = pg + kHdrBytes + (2 + cb) * P;
  r.rs = lds16(rsec + 2 * rA) | (lds16(rsec + 2 * rB) << 16);
  r.vs = lds16(ssec + 2 * rA) | (lds16(ssec + 2 * rB) << 16);
  const uint32_t vsec = pg + kHdrBytes + (2 + cb + 2) * P + (row0 >> 3) * 1024;
  const uint4 xa = lds128(vsec + lane * 16), ya = lds128(vsec + 512 + lane * 16);
  const uint4 xb = lds128(vsec + 1024 + lane * 16), yb = lds128(vsec + 1536 + lane * 16);
  r.va[0] = xa.x; r.va[1] = xa.y; r.va[2] = xa.z; r.va[3] = xa.w;
  r.va[4] = ya.x; r.va[5] = ya.y; r.va[6] = ya.z; r.va[7] = ya.w;
  r.vb[0] = xb.x; r.vb[1] = xb.y; r.vb[2] = xb.z; r.vb[3] = xb.w;
  r.vb[4] = yb.x; r.vb[5] = yb.y; r.vb[6] = yb.z; r.vb[7] = yb.w;
}

// T1 logits from code words in registers (see logits_t1)
__device__ __forceinline__ void logits_t1_regs(const uint32_t (&wa)[4], const uint32_t (&wb)[4],
                                               uint32_t tb, const QFrag& f, float (&c)[4],
                                               float (&d)[4]) {
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int i = s >> 1, k0 = 2 * (s & 1);
    const uint32_t ea0 = lds32(t1_addr(wa[i], k0, tb)), ea1 = lds32(t1_addr(wa[i], k0 + 1, tb));
    const uint32_t eb0 = lds32(t1_addr(wb[i], k0, tb)), eb1 = lds32(t1_addr(wb[i], k0 + 1, tb));
    if (s & 1)
      mma_k16<false>(d, ea0, eb0, ea1, eb1, f.b[2 * s], f.b[2 * s + 1]);
    else
      mma_k16<false>(c, ea0, eb0, ea1, eb1, f.b[2 * s], f.b[2 * s + 1]);
  }
}

// T2 logits from code words in registers (see logits_t2)
__device__ __forceinline__ void logits_t2_regs(const uint32_t (&wa)[4], const uint32_t (&wb)[4],
                                               uint32_t tb, const QFrag& f, float (&c)[4],
                                               float (&d)[4]) {
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const uint32_t ea0 = lds32(t2_addr(wa[0], wa[1], wa[2], 2 * s, tb));
    const uint32_t ea1 = lds32(t2_addr(wa[0], wa[1], wa[2], 2 * s + 1, tb));
    const uint32_t eb0 = lds32(t2_addr(wb[0], wb[1], wb[2], 2 * s, tb));
    const uint32_t eb1 = lds32(t2_addr(wb[0], wb[1], wb[2], 2 * s + 1, tb));
    if (s & 1)
      mma_k16<false>(d, ea0, eb0, ea1, eb1, f.b[2 * s], f.b[2 * s + 1]);
    else
      mma_k16<false>(c, ea0, eb0, ea1, eb1, f.b[2 * s], f.b[2 * s + 1]);
  }
}

// 16 T1 / T2 rows [row0, row0 + 16) from their loaded ring data.
template <int G, bool CAP>
__device__ __forceinline__ void compute_code_rows(const DecodeParams& p, const CodeRows& r,
                                                  uint32_t tier, int row0, const QFrag& qf,
                                                  uint32_t tb1, uint32_t tb2, WarpState& st,
                                                  int lane, float* lg) {
  const int t = lane >> 2, g = lane & 3;
  const uint32_t cnt = r.hdr & 0xFFFFu;
  if ((r.hdr >> 16) != (tier | ((uint32_t)kPageMagic << 8)) || cnt > (uint32_t)p.P) {
    if (lane == 0) report(p.err, SKV_ERR_CORRUPT);
    return;
  }
  if ((uint32_t)row0 >= cnt) return;
  const int rA = row0 + t, rB = rA + 8;
  const bool vA = (uint32_t)rA < cnt, vB = (uint32_t)rB < cnt;
  float c[4] = {0.0f, 0.0f, 0.0f, 0.0f}, d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  if (tier == SKV_TIER_T1)
    logits_t1_regs(r.ca, r.cb, tb1, qf, c, d);
  else
    logits_t2_regs(r.ca, r.cb, tb2, qf, c, d);
  const float a = c[0] + d[0], b = c[2] + d[2];
  const float rtA = __half2float(__ushort_as_half((unsigned short)(r.rs & 0xFFFFu)));
  const float rtB = __half2float(__ushort_as_half((unsigned short)(r.rs >> 16)));
  const float vsA = __half2float(__ushort_as_half((unsigned short)(r.vs & 0xFFFFu)));
  const float vsB = __half2float(__ushort_as_half((unsigned short)(r.vs >> 16)));
  const float lA = vA ? a * (rtA * qf.c1) : -INFINITY;
  const float lB = vB ? b * (rtB * qf.c1) : -INFINITY;
  if constexpr (CAP) capture_logits<G>(lg, rA, rB, vA, vB, lA, lB, g);
  uint32_t bf0, bf1;
  softmax_weights<G, true>(lA, lB, vA ? vsA : 0.0f, vB ? vsB : 0.0f, st, lane, bf0, bf1);
  pv_int8_regs(r.va, r.vb, bf0, bf1, st);
}

template <int G, bool DENSE, bool CAP, int VAR>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    decode_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  using Smem = DecodeSmem<G, DENSE>;
  const uint32_t base = smem_u32(smem_raw);
  const uint32_t limit = base + (uint32_t)p.smem_bytes;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const int U = p.B * p.Hkv;
  SplitInfo si;
  si.indptr = p.indptr;
  si.tier_indptr = p.tier_indptr;
  si.U = U;
  si.w[0] = p.cost[0];
  si.w[1] = DENSE ? p.cost[0] : p.cost[1];
  si.w[2] = DENSE ? p.cost[0] : p.cost[2];
  const DecodeWs wsl = decode_ws(p.S, U, G);
  uint8_t* const wsb = reinterpret_cast<uint8_t*>(p.part);
  int* const counters = reinterpret_cast<int*>(wsb + wsl.ctr);
  const int ipp = kItemRows >> p.log2P;
  // the largest item: ipp pages of the largest payload
  int maxpay = p.payload[0];
  if (!DENSE) maxpay = max(maxpay, max(p.payload[1], p.payload[2]));
  uint32_t ring_lo, R, tbl1, fixed_at;
  const bool plan_ok = smem_layout<G, DENSE>(base, limit, (uint32_t)sizeof(Smem),
                                             (uint32_t)(ipp * maxpay), ring_lo, R, tbl1, fixed_at);
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + (plan_ok ? fixed_at - base : 0u));

  if (tid == 0) {
    if (plan_ok) {
      for (int i = 0; i < kNSlot; ++i) {
        mbar_init(smem_u32(&sm.full[i]), 1);
        mbar_init(smem_u32(&sm.empty[i]), kGW);
        mbar_init(smem_u32(&sm.ready[i]), 1);
      }
      sm.abort_flag = 0;
      sm.dyn_go = 0;
      fence_mbar_init();
    } else {
      report(p.err, SKV_ERR_ARG);
    }
  }
  // the merge kernel may be launched now: it waits for this grid's end
  asm volatile("griddepcontrol.launch_dependents;");
  if (tid == kDecodeThreads - 1) {
    // CTA c brings slice c of the queries into L2 (the consumers load their
    // unit's heads once the split is known)
    const long long lines = ((long long)p.B * p.Hq * kHeadDim * 2 + 127) / 128;
    for (long long l = lines * c / p.S; l < lines * (c + 1) / p.S; ++l)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const uint8_t*>(p.q) + 128 * l));
  }
  // units without any resident page: out = 0, lse = -inf, nothing to merge
  // (written by CTA 0, once the grids this one depends on have completed)
  if (c == 0) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int u = warp; u < U; u += kDecodeThreads / 32) {
      if (p.indptr[u + 1] > p.indptr[u]) continue;
      const long long o = (long long)(u / p.Hkv) * p.Hq + (long long)(u % p.Hkv) * G;
      for (int i = lane; i < G * kHeadDim; i += 32) p.out[o * kHeadDim + i] = 0.0f;
      if (p.lse && lane < G) p.lse[o + lane] = -INFINITY;
      if (lane == 0) reinterpret_cast<int2*>(counters)[u] = make_int2(0, 0);
    }
  }
  if (!plan_ok) return;  // uniform: every thread computed the same layout
  find_run(si, c, p.S, sm, tid, p.ids, ipp, p.dynamic != 0);
  const long long g0 = sm.run[0], g1 = sm.run[1];
  if (g0 >= g1) {
    // an empty run inside a unit's runs (unit-aligned: a trailing run of a
    // small unit; global: a run between two pages of one unit, when a page
    // costs more than a run) leaves an empty partial in its slot
    const int u = sm.unit0;
    const bool inside = unit_aligned_split(U, p.S) ? true
                                                  : (g0 < (long long)p.indptr[U] && g0 > (long long)p.indptr[u]);
    if (inside && tid < G) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      float* part = p.part + (long long)(c + u) * G * kPartStride + tid * kPartStride;
      part[0] = -INFINITY;
      part[1] = 0.0f;
      // (a unit's first run always holds pages; should it not, the counter
      // of the unit's chunks is still reset here, after the wait)
      if (tid == 0 && sm.dyn_chunks > 0 && sm.dyn_first)
        atomicExch(reinterpret_cast<unsigned long long*>(wsb + wsl.dyn) + u,
                   (unsigned long long)launch_tag() << 32);
    }
    return;
  }

  const int u0 = sm.unit0;  // the unit holding page g0

  if (warp == kPlannerWarp) {
    // ------------------------------------------------------------- planner
    // The run is planned as page ranges inside one unit each: the run's part
    // of every unit it touches (in order) and, under the unit-aligned split,
    // the dynamic chunks this CTA takes from its unit's counter once its
    // static part is planned.  A range is planned in batches of up to 32
    // items: lane i decodes item it + i (its page ids -> sources, sizes,
    // tiers) in parallel.  Placement is deterministic: an item goes at the
    // write offset, or at 0 when it would cross the ring's end.  Before an
    // item is published every older item whose bytes it may overwrite
    // (virtual start < its virtual end - R) and the previous user of its
    // slot must be released; each lane works out that count, and the lanes
    // publish (descriptors + ready signal) in parallel as releases arrive.
    // A unit's items are followed by kCG unit-end markers (one per consumer
    // group, no bytes) that carry the index of the next unit's first item;
    // the run ends with kIss end-of-run markers, one per issuer.
    const bool in_unit = unit_aligned_split(U, p.S);
    const int dyn_chunks = in_unit ? sm.dyn_chunks : 0;
    const long long dyn_m = sm.dyn_m;
    const int dyn_cp = sm.dyn_cp;
    int it = 0;                 // next item
    int tail = 0;               // oldest item not known to be released
    uint32_t wr = 0;            // ring write offset
    unsigned long long V = 0;   // virtual position of the write offset (grows by laps of R)
    bool ok = true;
    // wait until item `tail` is released, then advance tail
    auto release_tail = [&]() -> bool {
      if (!mbar_wait_bounded(smem_u32(&sm.empty[tail % kNSlot]), (uint32_t)((tail / kNSlot) & 1),
                             &sm.abort_flag, p.wait_limit))
        return false;
      ++tail;
      return true;
    };
    // a marker item (no bytes, no copy) in the next slot
    auto publish_marker = [&](uint32_t meta, uint32_t z, uint32_t bytes) -> bool {
      while (it - tail >= kNSlot)
        if (!release_tail()) return false;
      const int s = it % kNSlot;
      if (lane == 0) {
        sm.vstart[it & 63] = V;
        sm.desc[s] = make_uint4(0u, meta, z, 0u);
        sm.copy_bytes[s] = bytes;
        mbar_arrive(smem_u32(&sm.ready[s]));
      }
      __syncwarp();
      ++it;
      return true;
    };
    // the dynamic chunk counter of this run's unit: a grab returns {tag,
    // index}; a tag other than this launch's means the counter was not
    // reset yet (the grab is void)
    unsigned long long* const dynctr = reinterpret_cast<unsigned long long*>(wsb + wsl.dyn) + u0;
    const uint32_t tag = launch_tag();
    unsigned long long fut = 0;  // lane 0: the result of the grab in flight
    bool grabbed = false;
    bool grab_ok = true;
    auto issue_grab = [&]() {
      if (!grabbed) {
        // the first grab waits until the consumers have passed the wait for
        // the previous grids (no earlier launch still takes chunks from this
        // workspace) and, in the unit's first run, reset the counter
        const long long t0 = clock64();
        while (ld_volatile(&sm.dyn_go) == 0) {
          if (ld_volatile(&sm.abort_flag) || clock64() - t0 > p.wait_limit) {
            grab_ok = false;  // no grab: fut stays 0, whose tag matches no launch
            break;
          }
          __nanosleep(256);
        }
        grabbed = true;
      }
      if (grab_ok && lane == 0) fut = atomicAdd(dynctr, 1ull);
    };
    // the page ids of the unit's dynamic part, brought into L2 when the
    // static part is planned (the chunks' first id loads then hit L2)
    auto prefetch_dyn_ids = [&]() {
      // the 128-byte lines that hold ids [dyn_m, dyn_m + chunks * cp)
      const uintptr_t a = reinterpret_cast<uintptr_t>(p.ids + dyn_m);
      const uintptr_t l0 = a / 128, l1 = (a + (uintptr_t)dyn_chunks * dyn_cp * 4 + 127) / 128;
      for (uintptr_t l = l0 + lane; l < l1; l += 32)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const void*>(128 * l)));
    };
    // plan the items of pages [pg, pe) of one unit
    auto plan_range = [&](long long pg, long long pe, bool grab_at_last) -> bool {
      uint32_t idn[kMaxIPP];
#pragma unroll
      for (int q = 0; q < kMaxIPP; ++q) {
        const long long pq = pg + (long long)lane * ipp + q;
        idn[q] = (q < ipp && pq < pe) ? __ldg(p.ids + pq) : 0u;
      }
      while (pg < pe) {
        const int nb = (int)min(32LL, (pe - pg + ipp - 1) / ipp);  // items in this batch
        const long long pn = min(pe, pg + (long long)nb * ipp);    // the next batch's first page
        if (grab_at_last && pn >= pe) {  // the range's last batch: the first chunk's grab
          issue_grab();
          prefetch_dyn_ids();
        }
        const uint32_t my_pg = CAP ? (uint32_t)(pg + (long long)lane * ipp) : 0u;
        // ---- lane-parallel decode of item it + lane
        uint32_t plo[kMaxIPP], phi[kMaxIPP], psz[kMaxIPP];
        uint32_t total = 0, imeta = 0, relz = 0, relw = 0;
        uint32_t id[kMaxIPP];
#pragma unroll
        for (int q = 0; q < kMaxIPP; ++q) id[q] = idn[q];
#pragma unroll
        for (int q = 0; q < kMaxIPP; ++q) {
          const long long pq = pn + (long long)lane * ipp + q;
          idn[q] = (q < ipp && pq < pe) ? __ldg(p.ids + pq) : 0u;
        }
        if (lane < nb) {
          const long long ps = pg + (long long)lane * ipp;
          const int n = (int)min((long long)ipp, pe - ps);
          imeta = (uint32_t)n;
#pragma unroll
          for (int q = 0; q < kMaxIPP; ++q) {
            plo[q] = 0;
            phi[q] = 0;
            psz[q] = 0;
            if (q == 1) relz = total;
            if (q == 2) relz |= total << 16;
            if (q == 3) relw = total;
            if (q < n) {
              const uint32_t tr = id[q] >> 30, slot = id[q] & 0x3FFFFFFFu;
              bool valid;
              if (DENSE) {
                valid = tr == 0 && slot < (unsigned long long)p.slots[0];
              } else {
                valid = (tr == 0 && slot < (unsigned long long)p.slots[0]) ||
                        (tr == 1 && slot < (unsigned long long)p.slots[1]) ||
                        (tr == 2 && slot < (unsigned long long)p.slots[2]);
              }
              if (valid) {
                const uint8_t* src = tr == 0 ? p.pool[0] + (long long)slot * p.stride[0]
                                             : (tr == 1 ? p.pool[1] + (long long)slot * p.stride[1]
                                                        : p.pool[2] + (long long)slot * p.stride[2]);
                plo[q] = (uint32_t)reinterpret_cast<uintptr_t>(src);
                phi[q] = (uint32_t)(reinterpret_cast<uintptr_t>(src) >> 32);
                psz[q] = (uint32_t)(tr == 0 ? p.payload[0] : (tr == 1 ? p.payload[1] : p.payload[2]));
              } else {
                report(p.err, SKV_ERR_CORRUPT);
                imeta |= 1u << (kMetaBadShift + q);
              }
              imeta |= (tr & 3u) << (kMetaTierShift + 2 * q);
              total += psz[q];
            }
          }
        }
        // ---- placement: a warp-parallel scan of the sizes, then each lane
        // finds how many items must be released before its item may be
        // written (need: all items before it), and the lanes publish in
        // parallel, a prefix of the batch at a time, as releases come in
        uint32_t my_off = 0;
        unsigned long long my_v = 0;
        {
          // offsets = write offset + exclusive prefix of the sizes, restarted
          // at 0 (after a pad to the next lap of the virtual position) at the
          // first item of each stretch that would cross the ring's end
          uint32_t incl = total;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += y;
          }
          const uint32_t excl = incl - total;
          uint32_t base = wr;
          unsigned long long vbase = V;
          int from = 0;
          while (true) {
            const uint32_t ex0 = __shfl_sync(0xFFFFFFFFu, excl, from);
            const uint32_t off = base + (excl - ex0);
            const unsigned cross =
                __ballot_sync(0xFFFFFFFFu, lane >= from && lane < nb && off + total > R);
            const int j = cross ? __ffs(cross) - 1 : 32;
            if (lane >= from && lane < j) {
              my_off = off;
              my_v = vbase + (excl - ex0);
            }
            if (!cross) break;
            const uint32_t exj = __shfl_sync(0xFFFFFFFFu, excl, j);
            vbase = vbase + (exj - ex0) + (R - (base + (exj - ex0)));
            base = 0;
            from = j;
          }
          const uint32_t lt = __shfl_sync(0xFFFFFFFFu, total, nb - 1);
          wr = __shfl_sync(0xFFFFFFFFu, my_off, nb - 1) + lt;
          V = __shfl_sync(0xFFFFFFFFu, my_v, nb - 1) + lt;
        }
        if (lane < nb) sm.vstart[(it + lane) & 63] = my_v;
        __syncwarp();
        int need = 0;
        if (lane < nb) {
          const int me = it + lane;
          // slot reuse: item me - kNSlot must be released
          need = max(0, me - kNSlot + 1);
          // space: every item whose bytes start more than R before this
          // item's end (V grows with the item index: a prefix of them)
          const unsigned long long lim = my_v + total;
          // binary search: the first j in [need, me) with vstart[j] + R >= lim
          int lo = need, hi = me;
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (sm.vstart[mid & 63] + R >= lim) hi = mid; else lo = mid + 1;
          }
          need = lo;
        }
        bool done = lane >= nb;
        while (true) {
          // released items, in order, without blocking
          while (tail < it + nb &&
                 mbar_test_wait(smem_u32(&sm.empty[tail % kNSlot]), (uint32_t)((tail / kNSlot) & 1)))
            ++tail;
          const bool now = !done && need <= tail;
          if (now) {
            const int s = (it + lane) % kNSlot;
            sm.desc[s] = make_uint4(ring_lo + my_off, imeta, relz, relw);
            if (CAP) sm.dpage[s] = my_pg;
            const uint32_t rel[kMaxIPP] = {0u, relz & 0xFFFFu, relz >> 16, relw};
#pragma unroll
            for (int q = 0; q < kMaxIPP; ++q)
              if (q < (int)(imeta & 7u))
                sm.copy[s][q] = PageCopy{plo[q], phi[q], psz[q], ring_lo + my_off + rel[q]};
            sm.copy_bytes[s] = total;
            mbar_arrive(smem_u32(&sm.ready[s]));
          }
          done = done || now;
          if (__all_sync(0xFFFFFFFFu, done)) break;
          // the oldest unreleased item is published (its own need is met):
          // sleep until it is released
          if (!release_tail()) return false;
        }
        it += nb;
        pg = pn;
      }
      return true;
    };

    int u = u0;
    long long pg = g0;
    // end of the current unit's part of the run and the end of the next
    // unit, loaded one unit ahead (a unit-aligned run lies inside its unit)
    long long ub = in_unit ? g1 : min(g1, (long long)p.indptr[u0 + 1]);
    long long ub_next = (!in_unit && u0 + 2 <= U) ? (long long)p.indptr[u0 + 2] : g1;
    // One loop, one call of plan_range (so that it is inlined and the
    // planner's state stays in registers): each pass plans one range, the
    // run's part of the next unit or, after a unit's static part, the next
    // dynamic chunk grabbed (one grab in flight ahead of the chunk being
    // planned).  A unit ends with one marker per consumer group, carrying
    // the index of the next unit's first item.
    bool chunks = false;  // the current unit's static part is planned: take chunks
    while (ok) {
      long long rs, re;
      bool grab_last = false, unit_end = false;
      if (chunks) {
        const unsigned long long got = __shfl_sync(0xFFFFFFFFu, fut, 0);
        const uint32_t k = (uint32_t)got;
        if ((uint32_t)(got >> 32) != tag || k >= (uint32_t)dyn_chunks) {
          chunks = false;
          const uint32_t next_first = (uint32_t)(it + kCG);
          for (int e = 0; e < kCG && ok; ++e) ok = publish_marker(kMetaUnitEnd, next_first, 0u);
          continue;
        }
        issue_grab();
        rs = dyn_m + (long long)k * dyn_cp;
        re = rs + dyn_cp;
      } else {
        if (pg >= g1) break;
        while (pg >= ub) {  // next unit with pages in this run
          ++u;
          ub = min(g1, ub_next);
          ub_next = u + 2 <= U ? (long long)p.indptr[u + 2] : g1;
        }
        rs = pg;
        re = ub;
        pg = ub;
        grab_last = dyn_chunks > 0;
        chunks = dyn_chunks > 0;
        unit_end = !chunks;
      }
      ok = plan_range(rs, re, grab_last);
      if (ok && unit_end) {
        const uint32_t next_first = (uint32_t)(it + kCG);
        for (int e = 0; e < kCG && ok; ++e) ok = publish_marker(kMetaUnitEnd, next_first, 0u);
      }
    }
    // end-of-run markers: a slot each (its previous item released)
    for (int e = 0; e < kIss && ok; ++e) ok = publish_marker(0u, 0u, kEndOfRun);
    if (lane == 0 && !ok) {
      report(p.err, SKV_ERR_TIMEOUT);
      sm.abort_flag = 1;
    }
    return;
  }
  if (warp > kPlannerWarp) {
    // ------------------------------------------------------------- issuers
    if (lane != 0) return;
    const int k = warp - kPlannerWarp - 1;
    int it = k;
    bool ok = true;
    while (true) {
      const int s = it % kNSlot;
      if (!mbar_wait_bounded(smem_u32(&sm.ready[s]), (uint32_t)((it / kNSlot) & 1),
                             &sm.abort_flag, p.wait_limit)) {
        ok = false;
        break;
      }
      const uint32_t total = sm.copy_bytes[s];
      if (total == kEndOfRun) break;
      const uint32_t np = sm.desc[s].y & 7u;
      const uint32_t fullb = smem_u32(&sm.full[s]);
      // the item's copy list is read before the arrive: once the phase can
      // complete (no bytes to wait for), the slot may be released and
      // rewritten for a later item
      PageCopy cps[kMaxIPP];
#pragma unroll
      for (int q = 0; q < kMaxIPP; ++q) {
        cps[q] = PageCopy{0u, 0u, 0u, 0u};
        if ((uint32_t)q < np) cps[q] = sm.copy[s][q];
      }
      mbar_arrive_expect_tx(fullb, total);
#pragma unroll
      for (int q = 0; q < kMaxIPP; ++q) {
        const PageCopy& cp = cps[q];
        if (cp.bytes)
          bulk_g2s(cp.dst, reinterpret_cast<const void*>((uintptr_t)cp.src_lo |
                                                         ((uintptr_t)cp.src_hi << 32)),
                   cp.bytes, fullb);
      }
      it += kIss;
    }
    if (!ok) {
      report(p.err, SKV_ERR_TIMEOUT);
      sm.abort_flag = 1;
      // let every copy this issuer started land before the CTA can exit
      // (with the fixed ~1 s limit, whatever the run-time wait limit: no CTA
      // may leave with a copy into its shared memory in flight)
      const long long t0 = clock64();
      for (int jj = it - kIss; jj >= 0 && jj >= it - kNSlot; jj -= kIss) {
        while (!mbar_try_wait(smem_u32(&sm.full[jj % kNSlot]), (uint32_t)((jj / kNSlot) & 1)) &&
               clock64() - t0 < kWaitLimitCycles) {
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  // A failed (timed-out) wait never breaks the loops: every consumer warp
  // must run the same sequence of named barriers.  After a failure the CTA's
  // abort flag makes every later wait return at once and work is skipped.
  const int nct = kNCW * 32;
  const int t4 = lane & 3, gq = lane >> 2;
  const int grp = warp / kGW, wi = warp % kGW;  // consumer group, warp within it
  // this lane's copy in the reconstruction tables; TBL1's space doubles as
  // the stash of the combine (then rebuilt before the next unit)
  const uint32_t tb1 = tbl1 + (uint32_t)lane * 4u, tb2 = tb1 + kTbl1;
  uint8_t* const tbl1p = smem_raw + (tbl1 - base);
  float* const stashp = reinterpret_cast<float*>(tbl1p);
  static_assert(DENSE || kNCW * 4 * kStashRow * 4 <= (int)kTbl1, "combine stash fits TBL1");
  // The decode may be a programmatic dependent of the previous step's grids
  // (launched while they finish).  The planner and the issuers start on the
  // page table and the pages at once: the store is never written by a grid
  // that lets dependents start early.  The consumers build the code tables
  // (parameters only), then wait for those grids before they read the
  // queries or write any result or partial.
  if constexpr (!DENSE) build_tables<VAR>(p, tbl1p, 256 + 64, tid, nct);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) {
    // the previous grids have completed: no earlier launch takes chunks from
    // this workspace any more.  The unit's first run resets its counter to
    // this launch's tag; then the planner may grab.
    if (sm.dyn_chunks > 0 && sm.dyn_first && unit_aligned_split(U, p.S)) {
      unsigned long long* ctr = reinterpret_cast<unsigned long long*>(wsb + wsl.dyn) + u0;
      atomicExch(ctr, (unsigned long long)launch_tag() << 32);
      __threadfence();
    }
    *reinterpret_cast<volatile int*>(&sm.dyn_go) = 1;
  }
  int tbl_entries = 0;  // table entries still to build (after a combine's stash)
  int it = 0;  // item index within the run
  bool ok = true;
  constexpr int kQPer = (4 * kHeadDim + kNCW * 32 - 1) / (kNCW * 32);  // q elements per thread
  for (int u = u0; u < U; ++u) {
    const int bb = u / p.Hkv, hkv = u % p.Hkv;
    // the unit's page range and its query elements, loaded together
    const long long iu0 = p.indptr[u], iu1 = p.indptr[u + 1];
    uint16_t qraw[kQPer];
#pragma unroll
    for (int k = 0; k < kQPer; ++k) {
      const int i = tid + k * nct;
      qraw[k] = i < G * kHeadDim
                    ? reinterpret_cast<const uint16_t*>(p.q)[((long long)bb * p.Hq + (long long)hkv * G) *
                                                                 kHeadDim + i]
                    : (uint16_t)0;
    }
    if (iu0 >= g1) break;
    const long long a = max(g0, iu0), b = min(g1, iu1);
    if (a >= b) continue;
    named_bar_sync(1, nct);
    if (tid < 4) sm.useg[tid] = si.seg_start(3 * u + tid);
    const bool many_units = sm.unit1 - sm.unit0 >= kTouchedUnits;
    if (many_units) {
      // many units in this run: the cost before unit u, summed afresh
      unsigned long long part = 0;
      for (int k = tid; k < 3 * u; k += nct)
        part += (unsigned long long)(si.seg_start(k + 1) - si.seg_start(k)) * si.weight(k);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, o);
      if (lane == 0) sm.scan[warp] = part;
    }
#pragma unroll
    for (int k = 0; k < kQPer; ++k) {
      const int i = tid + k * nct;
      if (i < G * kHeadDim) {
        const int h = i / kHeadDim, d = i % kHeadDim;
        sm.q32[h][d] = p.q_bf16 ? __bfloat162float(__ushort_as_bfloat16(qraw[k]))
                                : __half2float(__ushort_as_half(qraw[k]));
        if constexpr (DENSE) sm.O[h][d] = 0.0f;
      }
    }
    if constexpr (!DENSE) {
      if (tbl_entries) build_tables<VAR>(p, tbl1p, tbl_entries, tid, nct);
      tbl_entries = 0;
    }
    named_bar_sync(1, nct);
    if (tid == 0) {
      // the runs that hold this unit's partials, c0 .. c1 (read by the
      // combine, after its barriers): unit-aligned split, [B(u), B(u + 1));
      // global split, the runs of u's first and last page, run c holding
      // page g when floor(C(g) S / total) == c.  Computed now, while the
      // first items are in flight, to keep the divisions off the tail.
      unsigned long long cu[4];
      if (!many_units) {
#pragma unroll
        for (int t = 0; t < 4; ++t) cu[t] = sm.ucost[3 * (u - sm.unit0) + t];
      } else {
        unsigned long long cb = 0;
        for (int w2 = 0; w2 < kNCW; ++w2) cb += sm.scan[w2];
        cu[0] = cb;
#pragma unroll
        for (int t = 0; t < 3; ++t)
          cu[t + 1] = cu[t] + (unsigned long long)(sm.useg[t + 1] - sm.useg[t]) * si.weight(t);
      }
      const unsigned long long ctot = sm.ctot, Su = (unsigned long long)p.S;
      int c0 = c, c1 = c;
      if (unit_aligned_split(U, p.S)) {
        c0 = unit_first_run(u, cu[0], ctot, p.S, U);
        c1 = unit_first_run(u + 1, cu[3], ctot, p.S, U) - 1;
      } else if (ctot > 0) {
        int tl = 2;  // tier of the unit's last page
        while (tl > 0 && sm.useg[tl] == iu1) --tl;
        c0 = (int)udiv64(cu[0] * Su, ctot);
        c1 = (int)udiv64((cu[3] - si.weight(tl)) * Su, ctot);
      }
      sm.c01[0] = c0;
      sm.c01[1] = c1;
    }
    QFrag qf;
    make_qfrag<G, DENSE>(sm.q32, p.qk_scale_log2, p.q_bf16 != 0, lane, qf);
    WarpState st;
    st.m = kNoMax;
    st.l = 0.0f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) st.acc[mt][e] = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) st.ones[e] = 0.0f;

    // this group's items of the unit, it + i with (it + i) % kCG == grp, up
    // to its unit-end marker (which gives the next unit's first item)
    int next_it = it;
    for (int itm = it + ((grp - it % kCG) + kCG) % kCG; ok; itm += kCG) {
      const int s = itm % kNSlot;
      const uint32_t par = (uint32_t)((itm / kNSlot) & 1);
      // first the item's publication, then its data.  A phase-parity wait
      // on `full` alone would alias: while the slot's previous item
      // (itm - kNSlot, another group's) is still in flight, `full` is one
      // phase behind and its parity test would already pass.  `ready` for
      // item itm cannot be behind (the planner publishes in order and this
      // group's previous item, itm - kCG, is published), and once itm is
      // published the slot's previous item has been released, so `full`
      // is then at itm's own phase.
      const uint32_t readyb = smem_u32(&sm.ready[s]), fullb = smem_u32(&sm.full[s]);
      if ((!mbar_test_wait(readyb, par) && !mbar_wait_bounded(readyb, par, &sm.abort_flag, p.wait_limit)) ||
          (!mbar_test_wait(fullb, par) && !mbar_wait_bounded(fullb, par, &sm.abort_flag, p.wait_limit))) {
        ok = false;
        if (lane == 0) {
          report(p.err, SKV_ERR_TIMEOUT);
          sm.abort_flag = 1;
        }
        break;
      }
      const uint4 d = lds128(smem_u32(&sm.desc[s]));
      if (d.y & kMetaUnitEnd) {
        next_it = (int)d.z;
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));
        break;
      }
      const uint32_t np = d.y & 7u;
      const long long dpg = CAP ? (long long)sm.dpage[s] : -1;
      bool released = false;
      static_assert(kPasses == 1, "one 16-row pass per warp and item");
      {
        const int r = kRowsPerWarp * wi;  // row within the item
        const uint32_t kp = (uint32_t)(r >> p.log2P);
        const int row0 = r & (p.P - 1);
        if (kp < np && !((d.y >> (kMetaBadShift + kp)) & 1u)) {
          const uint32_t rel = kp == 0 ? 0u
                                       : (kp == 1 ? (d.z & 0xFFFFu)
                                                  : (kp == 2 ? (d.z >> 16) : d.w));
          float* lg = nullptr;
          if (CAP && dpg >= 0) {
            const long long r0 = (dpg + kp) * p.P;  // the page's first logit row
            if (r0 + p.P <= p.logit_rows)
              lg = p.logits + r0 * G;
            else if (lane == 0)
              report(p.err, SKV_ERR_ARG);
          }
          const uint32_t tier = (d.y >> (kMetaTierShift + 2 * kp)) & 3u;
          if (!DENSE && (tier == SKV_TIER_T1 || tier == SKV_TIER_T2)) {
            // code rows: everything this warp reads of the ring goes to
            // registers first, then the warp releases its share of the item
            CodeRows cr;
            load_code_rows(d.x + rel, p.P, tier == SKV_TIER_T1, row0, lane, cr);
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));
            released = true;
            compute_code_rows<G, CAP>(p, cr, tier, row0, qf, tb1, tb2, st, lane, lg);
          } else {
            process_rows<G, DENSE, CAP, (VAR & 4) != 0>(p, d.x + rel, tier, row0, qf, tb1, tb2,
                                                        st, lane, lg, sm.q32);
          }
        }
      }
      __syncwarp();
      if (lane == 0 && !released) mbar_arrive(smem_u32(&sm.empty[s]));
    }
    it = next_it;

    // ---- combine the warps' states into this CTA's partial for unit u.
    // Every warp writes its (m, l) per head; one thread per head forms M,
    // L and the warps' weights 2^(m_w - M).  ADA: the warps' unscaled
    // accumulators go to a stash (TBL1's space, rebuilt before the next
    // unit) and each output is their weighted sum.  Dense (no tables): the
    // warps add their scaled accumulators into O with shared atomics.
    float l = st.l;
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 4);
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 8);
    l += __shfl_xor_sync(0xFFFFFFFFu, l, 16);
    if (lane < G) {
      sm.ml[warp][lane][0] = st.m <= kNoMax ? -INFINITY : st.m;  // no row seen: -inf
      sm.ml[warp][lane][1] = l;
    }
    if constexpr (DENSE) {
      named_bar_sync(1, nct);
      if (tid < G) {
        const int n = tid;
        float M = -INFINITY;
        for (int w = 0; w < kNCW; ++w) M = fmaxf(M, sm.ml[w][n][0]);
        float L = 0.0f;
        for (int w = 0; w < kNCW; ++w) {
          const float mw = sm.ml[w][n][0];
          const float sc = (mw == -INFINITY) ? 0.0f : exp2f(mw - M);
          sm.wsc[w][n] = sc;
          L += sm.ml[w][n][1] * sc;
        }
        sm.MH[n] = M;
        sm.LH[n] = M == -INFINITY ? 0.0f : L;
      }
      named_bar_sync(1, nct);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int n = 2 * t4 + j;
        if (n < G) {
          const float sc = sm.wsc[warp][n];
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            atomicAdd(&sm.O[n][16 * mt + gq], st.acc[mt][j] * sc);
            atomicAdd(&sm.O[n][16 * mt + gq + 8], st.acc[mt][2 + j] * sc);
          }
        }
      }
      named_bar_sync(1, nct);
    } else {
      // ADA: one thread per head forms M, L and the warps' scales while the
      // warps stash their unscaled accumulators in TBL1's space (rows of
      // kStashRow floats: the two heads a store instruction covers fall in
      // different banks); then every output is a kNCW-term dot product of
      // scales and stash, written straight to out or to the partial.
      named_bar_sync(1, nct);  // every warp is done with the items and the tables
      if (tid < G) {
        const int n = tid;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kNCW; ++w) M = fmaxf(M, sm.ml[w][n][0]);
        float L = 0.0f;
#pragma unroll
        for (int w = 0; w < kNCW; ++w) {
          const float mw = sm.ml[w][n][0];
          const float sc = (mw == -INFINITY) ? 0.0f : exp2f(mw - M);
          sm.wsc[w][n] = sc;
          L = fmaf(sm.ml[w][n][1], sc, L);
        }
        sm.MH[n] = M;
        sm.LH[n] = M == -INFINITY ? 0.0f : L;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int n = 2 * t4 + j;
        if (n < G) {
          const float bias = 1152.0f * st.ones[j];  // int8 V offset (see softmax_pv)
          float* stash = stashp + (warp * G + n) * kStashRow;
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            stash[16 * mt + gq] = st.acc[mt][j] - bias;
            stash[16 * mt + gq + 8] = st.acc[mt][2 + j] - bias;
          }
        }
      }
      tbl_entries = 256;  // TBL1 holds the stash now
      named_bar_sync(1, nct);
      const int c0 = sm.c01[0], c1 = sm.c01[1];
      const long long obase = (long long)bb * p.Hq + (long long)hkv * G;
      float* part = p.part + (long long)(c + u) * G * kPartStride;
      for (int i = tid; i < G * kHeadDim; i += nct) {
        const int n = i / kHeadDim, d = i % kHeadDim;
        float o = 0.0f;
#pragma unroll
        for (int w = 0; w < kNCW; ++w) o = fmaf(stashp[(w * G + n) * kStashRow + d], sm.wsc[w][n], o);
        const float L = sm.LH[n];
        if (c0 == c1) {
          p.out[(obase + n) * kHeadDim + d] = L > 0.0f ? o / L : 0.0f;
          if (d == 0 && p.lse)
            p.lse[obase + n] = L > 0.0f ? (sm.MH[n] + log2f(L)) * 0.69314718055994530942f : -INFINITY;
        } else {
          part[n * kPartStride + 4 + d] = o;
          if (d == 0) {
            part[n * kPartStride + 0] = sm.MH[n];
            part[n * kPartStride + 1] = L;
          }
        }
      }
      if (tid == 0 && c == c0) reinterpret_cast<int2*>(counters)[u] = make_int2(c0, c1);
      if (b == g1) break;  // the run ends in this unit: no further page-table reads
      continue;
    }
    // ---- dense: this CTA's result for unit u (sm.O, sm.MH, sm.LH).  A unit
    // inside one run is finished here; otherwise every run from c0 to c1
    // writes its partial to slot c + u (an empty run an empty one, at the
    // kernel's start) and decode_merge_kernel combines them once this grid
    // has completed.  The CTA of run c0 records (c0, c1) for it.
    const int c0 = sm.c01[0], c1 = sm.c01[1];
    const long long obase = (long long)bb * p.Hq + (long long)hkv * G;
    if (c0 == c1) {
      for (int i = tid; i < G * kHeadDim; i += nct) {
        const int n = i / kHeadDim, d = i % kHeadDim;
        const float L = sm.LH[n];
        p.out[(obase + n) * kHeadDim + d] = L > 0.0f ? sm.O[n][d] / L : 0.0f;
        if (d == 0 && p.lse)
          p.lse[obase + n] = L > 0.0f ? (sm.MH[n] + log2f(L)) * 0.69314718055994530942f : -INFINITY;
      }
    } else {
      float* part = p.part + (long long)(c + u) * G * kPartStride;
      for (int i = tid; i < G * kHeadDim; i += nct) {
        const int n = i / kHeadDim, d = i % kHeadDim;
        part[n * kPartStride + 4 + d] = sm.O[n][d];
        if (d == 0) {
          part[n * kPartStride + 0] = sm.MH[n];
          part[n * kPartStride + 1] = sm.LH[n];
        }
      }
    }
    if (tid == 0 && c == c0) reinterpret_cast<int2*>(counters)[u] = make_int2(c0, c1);
    if (b == g1) break;  // the run ends in this unit: no further page-table reads
  }
}

// Cross-CTA merge (log-sum-exp) of the units that span several runs: one
// CTA per unit, one thread per (head, output pair), launched behind the
// decode grid as a programmatic dependent (its wait returns once the decode
// grid has completed and its writes are visible).  A unit's record (c0, c1)
// names its runs; every run in that range wrote slot c + u.  The loads of a
// batch of runs are all in flight at once, with an online maximum across
// batches.
template <int G>
__global__ void __launch_bounds__(G * kHeadDim / 2)
    decode_merge_kernel(const __grid_constant__ DecodeParams p) {
  // a programmatic dependent of the merge (the utility update) may start
  // its own prologue now; it waits for this grid before reading results
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int u = blockIdx.x;
  const int U = p.B * p.Hkv;
  const DecodeWs wsl = decode_ws(p.S, U, G);
  const int2 rr = reinterpret_cast<const int2*>(reinterpret_cast<const uint8_t*>(p.part) + wsl.ctr)[u];
  const int c0 = rr.x, nr = rr.y - rr.x + 1;
  if (nr <= 1) return;
  const int n = threadIdx.x / (kHeadDim / 2), j = threadIdx.x % (kHeadDim / 2);
  const float* pn = p.part + (long long)(c0 + u) * G * kPartStride + n * kPartStride;
  float M = -INFINITY, L = 0.0f, ox = 0.0f, oy = 0.0f;
  for (int r0 = 0; r0 < nr; r0 += kMergeBatch) {
    float2 ml[kMergeBatch], v[kMergeBatch];
#pragma unroll
    for (int k = 0; k < kMergeBatch; ++k) {
      const bool live = r0 + k < nr;
      const float* pr = pn + (long long)(r0 + k) * G * kPartStride;
      ml[k] = live ? __ldcg(reinterpret_cast<const float2*>(pr)) : make_float2(-INFINITY, 0.0f);
      v[k] = live ? __ldcg(reinterpret_cast<const float2*>(pr + 4 + 2 * j)) : make_float2(0.0f, 0.0f);
    }
    float Mb = M;
#pragma unroll
    for (int k = 0; k < kMergeBatch; ++k) Mb = fmaxf(Mb, ml[k].x);
    if (Mb == -INFINITY) continue;  // nothing yet
    const float sc = (M == -INFINITY) ? 0.0f : exp2f(M - Mb);
    L *= sc;
    ox *= sc;
    oy *= sc;
#pragma unroll
    for (int k = 0; k < kMergeBatch; ++k) {
      // an empty partial (m = -inf) carries no l or o worth reading
      if (ml[k].x == -INFINITY) continue;
      const float wgt = exp2f(ml[k].x - Mb);
      L = fmaf(wgt, ml[k].y, L);
      ox = fmaf(wgt, v[k].x, ox);
      oy = fmaf(wgt, v[k].y, oy);
    }
    M = Mb;
  }
  const long long obase = (long long)(u / p.Hkv) * p.Hq + (long long)(u % p.Hkv) * G;
  float* o = p.out + (obase + n) * kHeadDim + 2 * j;
  o[0] = L > 0.0f ? ox / L : 0.0f;
  o[1] = L > 0.0f ? oy / L : 0.0f;
  if (j == 0 && p.lse)
    p.lse[obase + n] = L > 0.0f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
}

// Utility update: every position t < seq_lens[b] of every unit takes
// u <- gamma u + mass, where the mass of a resident token is its softmax
// weight summed over the G query heads of its kv head, 2^(l_g - lse_g log2 e)
// from the logit the decode captured for its row (page index in the unit's
// list * P + row, from row_of); dropped tokens have mass 0.  Grid: x over
// positions, y over units; one position per thread per pass, so the tier,
// row map and utility streams are read in position order (a tier segment's
// logit rows are in the same order).  Launched as a programmatic dependent
// of the merge: the loads that do not depend on the decode (tier, row map,
// old utility of the first position) are issued before the wait for the
// decode's results.  The unit's lse goes through shared memory: one load
// per block, not one per thread (the same 16 bytes requested by every
// thread would queue at a single L2 slice).
// One chunk of V consecutive positions of unit u: tier, row map and old
// utility (vector loads when V = 4: Tmax % 4 == 0 and the arrays aligned).
template <int V>
struct UtilChunk {
  uint32_t tr[V];
  int loc[V];
  float u_old[V];
};

template <int V>
__device__ __forceinline__ void load_chunk(const UtilityParams& p, long long at, UtilChunk<V>& c) {
  if constexpr (V == 4) {
    const uchar4 t = *reinterpret_cast<const uchar4*>(p.tier + at);
    const int4 l = *reinterpret_cast<const int4*>(p.row_of + at);
    const float4 u = *reinterpret_cast<const float4*>(p.utility + at);
    c.tr[0] = t.x; c.tr[1] = t.y; c.tr[2] = t.z; c.tr[3] = t.w;
    c.loc[0] = l.x; c.loc[1] = l.y; c.loc[2] = l.z; c.loc[3] = l.w;
    c.u_old[0] = u.x; c.u_old[1] = u.y; c.u_old[2] = u.z; c.u_old[3] = u.w;
  } else {
    c.tr[0] = p.tier[at];
    c.loc[0] = p.row_of[at];
    c.u_old[0] = p.utility[at];
  }
}

template <int G, int V>
__global__ void __launch_bounds__(256) utility_kernel(const UtilityParams p) {
  constexpr float kLog2e = 1.4426950408889634f;
  __shared__ float ls_s[G];
  // the next step's decode may start on the pages now (it waits for this
  // grid before reading queries or writing results; the store is not
  // written here)
  asm volatile("griddepcontrol.launch_dependents;");
  const int U = p.B * p.Hkv;
  const int T = (int)p.Tmax;
  bool waited = false;
  for (int u = blockIdx.y; u < U; u += gridDim.y) {
    const int len = min(T, p.seq_lens[u / p.Hkv]);
    const int nch = (len + V - 1) / V;  // chunks of V positions
    const long long base = (long long)u * T;
    const int c0 = blockIdx.x * blockDim.x + threadIdx.x;
    UtilChunk<V> ch;
    if (c0 < nch) load_chunk<V>(p, base + (long long)c0 * V, ch);
    if (!waited) {  // uniform: every thread of the block takes it on the first unit
      asm volatile("griddepcontrol.wait;" ::: "memory");
      waited = true;
    }
    __syncthreads();  // the previous unit's lse has been read
    if (threadIdx.x < G) ls_s[threadIdx.x] = __ldcg(p.lse + (long long)u * G + threadIdx.x) * kLog2e;
    __syncthreads();
    float ls2[G];
#pragma unroll
    for (int g = 0; g < G; ++g) ls2[g] = ls_s[g];
    const long long r0 = (long long)p.indptr[u] * p.P, r1 = (long long)p.indptr[u + 1] * p.P;
    for (int ci = c0; ci < nch; ci += gridDim.x * blockDim.x) {
      if (ci != c0) load_chunk<V>(p, base + (long long)ci * V, ch);
      // every resident position's logits are loaded before any is used
      float lv[V][G];
      bool live[V];
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int t = ci * V + v;
        const uint32_t tr = ch.tr[v];
        live[v] = t < len && tr != SKV_TIER_DROP;
#pragma unroll
        for (int g = 0; g < G; ++g) lv[v][g] = 0.0f;
        if (!live[v]) continue;
        const long long gr = r0 + ch.loc[v];
        if (tr > SKV_TIER_DROP || ch.loc[v] < 0 || gr >= r1 || gr >= p.logit_rows) {
          report(p.err, SKV_ERR_CORRUPT);  // the position keeps its old utility
          live[v] = false;
          continue;
        }
        const float* l = p.logits + gr * G;
        if constexpr (G == 4) {
          const float4 x = __ldcg(reinterpret_cast<const float4*>(l));
          lv[v][0] = x.x; lv[v][1] = x.y; lv[v][2] = x.z; lv[v][3] = x.w;
        } else if constexpr (G == 2) {
          const float2 x = __ldcg(reinterpret_cast<const float2*>(l));
          lv[v][0] = x.x; lv[v][1] = x.y;
        } else {
          lv[v][0] = __ldcg(l);
        }
      }
      float un[V];
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int t = ci * V + v;
        un[v] = ch.u_old[v];
        if (t >= len) continue;  // past the sequence: unchanged
        float mass = 0.0f;
        if (live[v]) {
#pragma unroll
          for (int g = 0; g < G; ++g) mass += exp2f(lv[v][g] - ls2[g]);
        } else if (ch.tr[v] != SKV_TIER_DROP) {
          continue;  // a corrupt row: unchanged
        }
        un[v] = p.gamma * ch.u_old[v] + mass;
      }
      if constexpr (V == 4)
        *reinterpret_cast<float4*>(p.utility + base + (long long)ci * 4) =
            make_float4(un[0], un[1], un[2], un[3]);
      else
        p.utility[base + ci] = un[0];
    }
  }
}

cudaError_t launch_utility(const UtilityParams& p, cudaStream_t stream) {
  const long long U = (long long)p.B * p.Hkv;
  if (U == 0 || p.Tmax == 0) return cudaSuccess;
  if (p.Tmax > (1LL << 30)) return cudaErrorInvalidValue;
  // four positions per thread when the rows of four are aligned vectors
  const bool vec = p.Tmax % 4 == 0 && (reinterpret_cast<uintptr_t>(p.tier) & 3) == 0 &&
                   (reinterpret_cast<uintptr_t>(p.row_of) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(p.utility) & 15) == 0;
  const long long V = vec ? 4 : 1;
  // about 2 waves of 256-thread blocks over all units, at least one block per unit
  const long long per_unit = std::max<long long>(1, (148LL * 8 * 2 + U - 1) / U);
  const long long bx = std::min<long long>((p.Tmax + 256 * V - 1) / (256 * V), per_unit);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)bx, (unsigned)std::min<long long>(U, 65535));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (vec) {
    switch (p.G) {
      case 1: return cudaLaunchKernelEx(&cfg, utility_kernel<1, 4>, p);
      case 2: return cudaLaunchKernelEx(&cfg, utility_kernel<2, 4>, p);
      case 4: return cudaLaunchKernelEx(&cfg, utility_kernel<4, 4>, p);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (p.G) {
    case 1: return cudaLaunchKernelEx(&cfg, utility_kernel<1, 1>, p);
    case 2: return cudaLaunchKernelEx(&cfg, utility_kernel<2, 1>, p);
    case 4: return cudaLaunchKernelEx(&cfg, utility_kernel<4, 1>, p);
    default: return cudaErrorInvalidValue;
  }
}

// Context-parallel combine: rank r attended over its own slice of every
// sequence's tokens and produced (out_r, lse_r) per (sequence, query head);
// the softmax over the union of the slices is out = sum_r w_r out_r /
// sum_r w_r, lse = M + log sum_r w_r with w_r = exp(lse_r - M), M the largest
// lse_r.  Empty partials (lse -inf) carry no weight; all empty: out 0,
// lse -inf.  One block of 64 threads per row, a float2 of out per thread.
__global__ void __launch_bounds__(64) merge_partials_kernel(int R, long long n,
                                                            const float* __restrict__ out_parts,
                                                            const float* __restrict__ lse_parts,
                                                            long long rank_stride,
                                                            float* __restrict__ out,
                                                            float* __restrict__ lse) {
  const long long row = blockIdx.x;
  const int j = threadIdx.x;
  float M = -INFINITY;
  for (int r = 0; r < R; ++r) M = fmaxf(M, __ldg(lse_parts + r * rank_stride + row));
  float L = 0.0f, ox = 0.0f, oy = 0.0f;
  if (M != -INFINITY) {
    for (int r = 0; r < R; ++r) {
      const float lr = __ldg(lse_parts + r * rank_stride + row);
      if (lr == -INFINITY) continue;  // an empty partial's out is never read
      const float w = expf(lr - M);
      const float2 o = __ldg(reinterpret_cast<const float2*>(out_parts + r * rank_stride +
                                                             row * kHeadDim) + j);
      L += w;
      ox = fmaf(w, o.x, ox);
      oy = fmaf(w, o.y, oy);
    }
  }
  float2* dst = reinterpret_cast<float2*>(out + row * kHeadDim) + j;
  *dst = L > 0.0f ? make_float2(ox / L, oy / L) : make_float2(0.0f, 0.0f);
  if (j == 0 && lse) lse[row] = L > 0.0f ? M + logf(L) : -INFINITY;
}

cudaError_t launch_merge_partials(int R, long long n, const float* out_parts,
                                  const float* lse_parts, long long rank_stride, float* out,
                                  float* lse, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  if (R <= 0 || n > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  merge_partials_kernel<<<(unsigned)n, kHeadDim / 2, 0, stream>>>(R, n, out_parts, lse_parts,
                                                                  rank_stride, out, lse);
  return cudaGetLastError();
}

template <int G, bool DENSE>
size_t decode_smem_fixed() {
  return ((sizeof(DecodeSmem<G, DENSE>) + 127) / 128) * 128;
}

template <int G, bool DENSE>
cudaError_t launch_decode_g(const DecodeParams& p, cudaStream_t stream, cudaEvent_t between) {
  const size_t smem = (size_t)p.smem_bytes;
  // the logit-capturing variant when a logits buffer is given (ADA only)
  const bool cap = !DENSE && p.logits != nullptr;
  // the code-table variant (ADA only; the dense pages have no codes):
  // bit 0 the T1 5 + 3 scheme, bit 1 the Lloyd-Max 2-bit share grid, bit 2
  // the fused T0 / bf16 path (alone: the API refuses it with bits 0 / 1)
  const int var = DENSE ? 0
                        : (p.t0_bf16 ? 4 : ((p.t1_scheme ? 1 : 0) | (p.share_grid ? 2 : 0)));
  using K = void (*)(const DecodeParams);
  K kern;
  if (DENSE) {
    kern = decode_kernel<G, DENSE, false, 0>;
  } else if (cap) {
    kern = var == 0 ? decode_kernel<G, DENSE, !DENSE, 0>
         : var == 1 ? decode_kernel<G, DENSE, !DENSE, 1>
         : var == 2 ? decode_kernel<G, DENSE, !DENSE, 2>
         : var == 3 ? decode_kernel<G, DENSE, !DENSE, 3>
                    : decode_kernel<G, DENSE, !DENSE, 4>;
  } else {
    kern = var == 0 ? decode_kernel<G, DENSE, false, 0>
         : var == 1 ? decode_kernel<G, DENSE, false, 1>
         : var == 2 ? decode_kernel<G, DENSE, false, 2>
         : var == 3 ? decode_kernel<G, DENSE, false, 3>
                    : decode_kernel<G, DENSE, false, 4>;
  }
  const int vi = (cap ? 1 : 0) + 2 * var;
  // The shared-memory opt-in is set once per device, variant and size
  // (outside any stream capture: the first call is expected to be eager).
  static size_t configured[10][64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || configured[vi][dev] < smem) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[vi][dev] = smem;
  }
  const int U = p.B * p.Hkv;
  {
    // a programmatic dependent of the stream's previous kernel: its CTAs may
    // start on the pages while that kernel finishes (see the kernel's waits)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.S);
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = (size_t)p.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return e;
  }
  if (between) {
    // a profile point right after the decode grid (an external record node
    // when the stream is being captured; the merge then follows it in order)
    e = cudaEventRecordWithFlags(between, stream, cudaEventRecordExternal);
    if (e != cudaSuccess) return e;
  }
  // the merge: a programmatic dependent of the decode grid (it may be
  // scheduled early and waits in-kernel for the grid's completion)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)U);
  cfg.blockDim = dim3(G * kHeadDim / 2);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_merge_kernel<G>, p);
  if (e != cudaSuccess) return e;
  return cudaSuccess;
}

template <int G, bool DENSE>
bool decode_plan_ok(int smem_bytes, int max_item) {
  // the dynamic shared window starts at offset 0 or after a 1 KB reserve
  for (uint32_t b = 0; b <= 1024; b += 1024) {
    uint32_t rlo, rsz, tbl1, fixed_at;
    if (!smem_layout<G, DENSE>(b, b + (uint32_t)smem_bytes, (uint32_t)sizeof(DecodeSmem<G, DENSE>),
                               (uint32_t)max_item, rlo, rsz, tbl1, fixed_at))
      return false;
  }
  return true;
}

bool decode_smem_ok(int G, bool dense, int smem_bytes, int max_item) {
  if (dense) {
    switch (G) {
      case 1: return decode_plan_ok<1, true>(smem_bytes, max_item);
      case 2: return decode_plan_ok<2, true>(smem_bytes, max_item);
      default: return decode_plan_ok<4, true>(smem_bytes, max_item);
    }
  }
  switch (G) {
    case 1: return decode_plan_ok<1, false>(smem_bytes, max_item);
    case 2: return decode_plan_ok<2, false>(smem_bytes, max_item);
    default: return decode_plan_ok<4, false>(smem_bytes, max_item);
  }
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
      case 1: return launch_decode_g<1, true>(p, stream, between);
      case 2: return launch_decode_g<2, true>(p, stream, between);
      case 4: return launch_decode_g<4, true>(p, stream, between);
    }
  } else {
    switch (G) {
      case 1: return launch_decode_g<1, false>(p, stream, between);
      case 2: return launch_decode_g<2, false>(p, stream, between);
      case 4: return launch_decode_g<4, false>(p, stream, between);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace skv
