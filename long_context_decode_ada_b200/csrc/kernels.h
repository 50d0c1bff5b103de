// kernels.h -- parameter blocks and launchers shared by the libskv .cu files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace skv {

constexpr int kPartStride = 132;  // floats per (partial, head): m, l, pad, pad, o[128]

struct DecodeParams {
  const void* q;
  int q_bf16;
  int B, Hq, Hkv;
  const int32_t* indptr;
  const int32_t* tier_indptr;  // [3U + 1] page offsets per (unit, tier) segment, or NULL
  const uint32_t* ids;
  const uint8_t* pool[3];
  long long slots[3];
  long long stride[3];
  int payload[3];
  int cost[3];          // split weight of a page of each tier (split_cost)
  float* out;
  float* lse;
  int32_t* err;
  float* part;
  float* logits;         // per-row log2-domain logits [rows][G], or NULL (no capture)
  long long logit_rows;  // rows the logits buffer holds (page_cap * P)
  int S;
  int P;
  int log2P;
  int smem_bytes;       // dynamic shared memory of the decode kernel
  float qk_scale_log2;  // log2(e) / sqrt(d)
  float cos6[64], sin6[64], cos4[16], sin4[16];
  float cos5[32], sin5[32];  // angles of the T1 variant (5-bit angle + 3-bit share)
  int t1_scheme;             // T1 code byte: 0 (angle6 << 2) | share2; 1 (angle5 << 3) | share3
  int share_grid;            // 2-bit share grid: 0 uniform, 1 Lloyd-Max
  int t0_bf16;               // T0 pages hold bf16 K / V (the fused T0 / bf16 path)
  int dynamic;               // unit-aligned split: hand out the units' last pages at run time
  long long wait_limit;      // SM clocks a planner / issuer / consumer wait may take
};

struct EncodeParams {
  const uint16_t* K;
  const uint16_t* V;
  int B, Hkv;
  long long Tmax;
  int P;
  const int32_t* seq_lens;
  const uint8_t* tier;
  const int32_t* row_of;
  const int32_t* indptr;
  const int32_t* tier_indptr;  // [3U + 1] page offsets per (unit, tier) segment, or NULL
  const uint32_t* ids;
  uint8_t* pool[3];
  long long slots[3];
  long long stride[3];
  int32_t* err;
  int dense_bf16;
  int t0_bf16;          // T0 rows as bf16 (the fused T0 / bf16 path)
  float bx6[64], by6[64], bx4[16], by4[16];
  float bx5[32], by5[32];
  int t1_scheme;        // 0: 6-bit angle + 2-bit share; 1: 5-bit angle + 3-bit share
  int share_grid;       // 2-bit share grid: 0 uniform, 1 Lloyd-Max
};

// Decode-time append of one token per sequence (every kv head) as T0.
struct AppendParams {
  const uint16_t* K;  // fp16 [B][Hkv][128]: the new token's keys
  const uint16_t* V;  // fp16 [B][Hkv][128]
  int B, Hkv;
  long long Tmax;
  int P;
  int32_t* seq_lens;        // [B], incremented
  uint8_t* tier;            // [B][Hkv][Tmax]
  int32_t* row_of;          // [B][Hkv][Tmax]
  int32_t* indptr;          // [U + 1], updated
  int32_t* tier_indptr;     // [3U + 1], updated
  uint32_t* ids;            // [page_cap], updated
  long long page_cap;
  uint8_t* pool0;           // the T0 pool
  long long slots0, stride0;
  const uint32_t* free0;    // T0 free slots, taken from *free0_cursor on
  long long free0_len;
  int32_t* free0_cursor;
  int32_t* err;
  int32_t* ws;              // append_ws() int32 words
  int t0_bf16;              // the T0 rows as bf16
};

// Append workspace (int32 words): per unit t, need, new-before, old T0 end;
// the old indptr [U + 1]; a flag word (1: the call changes nothing); the
// free-list cursor before the call; the number of new pages; the old page
// ids [page_cap] (copied only when pages are added).
struct AppendWs {
  size_t t, need, nb, a1, oindptr, flag, cur, total, oids, words;
};
__host__ __device__ inline AppendWs append_ws(long long U, long long page_cap) {
  AppendWs w;
  w.t = 0;
  w.need = w.t + (size_t)U;
  w.nb = w.need + (size_t)U;
  w.a1 = w.nb + (size_t)U;
  w.oindptr = w.a1 + (size_t)U;
  w.flag = w.oindptr + (size_t)U + 1;
  w.cur = w.flag + 1;
  w.total = w.cur + 1;
  w.oids = w.total + 1;
  w.words = w.oids + (size_t)page_cap;
  return w;
}

struct AllocParams {
  const uint16_t* K;
  int B, Hkv;
  long long Tmax;
  int P;
  const int32_t* seq_lens;
  const float* utility;
  const uint8_t* protect;
  int mode;
  const int64_t* budget;
  const int32_t* quota;
  const uint32_t* free_ids[3];
  long long free_len[3];
  uint8_t* pool[3];
  long long slots[3];
  long long stride[3];
  int payload[3];
  uint8_t* tier_out;
  int32_t* row_of;
  int32_t* indptr;
  int32_t* tier_indptr;       // [3U + 1] per (unit, tier) or NULL
  uint32_t* page_ids;
  long long page_cap;
  int32_t* err;
  float kappa[3];
  // workspace carve-up (device)
  float* keyw;                // [B*Hkv*Tmax]
  unsigned long long* sel;    // [nseg*3*3]: prefix, remaining (as u64), done
  unsigned long long* hist;   // [nseg*3*256]
  int32_t* counts;            // [U*3]
  int32_t* ccounts;           // [U][chunks of kRowChunk positions][3]: tier counts per chunk
  int32_t* tbase;             // [U*3]
  long long* pinned;          // [B]: bytes of the tokens whose tier is fixed
  int nseg;
  int dense;                  // dense-bf16 baseline packing (every token kept, tier 0)
  int outlier;                // outlier-aware protection on
  uint8_t* eff_protect;       // [B*Hkv*Tmax]: protect | outlier flag (workspace)
  // re-tiering (launch_retier_plan): the store as it was before the call,
  // snapshotted into the workspace, and the page bookkeeping of the update
  const uint8_t* demote;      // [B*Hkv*Tmax]: T0 rows to re-decide
  uint8_t* tier_old;          // [B*Hkv*Tmax]
  int32_t* row_old;           // [B*Hkv*Tmax]
  int32_t* indptr_old;        // [U + 1]
  int32_t* tindptr_old;       // [3U + 1]
  uint32_t* ids_old;          // [page_cap]
  int32_t* diff;              // [3U]: first row of each (unit, tier) segment that changes
  int32_t* keep;              // [3U]: leading pages of each segment kept in place
  int32_t* rbase;             // [U]: first released-list index of each unit
  int32_t* cursor;            // [3]: free-list cursors, advanced by the pages taken
  uint32_t* released;         // [page_cap]: ids of the old pages no longer referenced
  int32_t* n_released;        // [1]
};

// Decode workspace: partials [(S + U) G][kPartStride] fp32, then per unit the
// range (c0, c1) of runs that hold its partials (int32 pairs, written by every
// call before they are read), then per unit the 64-bit counter of the
// unit's dynamic chunks: {launch tag (high 32 bits), chunks handed out}, reset
// by the unit's first run of each launch (no state is kept between calls).
struct DecodeWs {
  size_t ctr, dyn, bytes;
};
__host__ __device__ inline DecodeWs decode_ws(long long S, long long U, int G) {
  DecodeWs w;
  w.ctr = (size_t)(S + U) * G * kPartStride * 4;
  w.dyn = w.ctr + 8 * (size_t)U;
  w.bytes = w.dyn + 8 * (size_t)U;
  return w;
}

size_t decode_fixed_smem(int G, bool dense);
// True when smem_bytes of dynamic shared memory hold the decode kernel's
// fixed block, LUTs and rings for items of up to max_item bytes.
bool decode_smem_ok(int G, bool dense, int smem_bytes, int max_item);
constexpr int kDecodeItemRows = 64;  // tokens per decode item
cudaError_t launch_decode(const DecodeParams& p, int G, bool dense, cudaStream_t stream,
                          cudaEvent_t between);

// Utility update from the captured logits and the merged lse of one decode.
struct UtilityParams {
  const float* logits;   // [rows][G] log2-domain logits written by the decode
  long long logit_rows;
  const float* lse;      // [B][Hq] natural-log lse of the decode
  const int32_t* seq_lens;
  const uint8_t* tier;   // [B][Hkv][Tmax]
  const int32_t* row_of; // [B][Hkv][Tmax]
  const int32_t* indptr; // [B*Hkv + 1]
  int B, Hkv, G, P;
  long long Tmax;
  float gamma;
  float* utility;        // [B][Hkv][Tmax] fp32, updated in place
  int32_t* err;
};
cudaError_t launch_utility(const UtilityParams& p, cudaStream_t stream);

// Log-sum-exp merge of R attention partials per (sequence, query head).
cudaError_t launch_merge_partials(int R, long long n, const float* out_parts,
                                  const float* lse_parts, long long rank_stride, float* out,
                                  float* lse, cudaStream_t stream);
cudaError_t launch_encode(const EncodeParams& p, cudaStream_t stream);
cudaError_t launch_append(const AppendParams& p, cudaStream_t stream);
constexpr int kRowChunk = 1024;  // positions per block of the count and row-map kernels
size_t alloc_workspace_bytes(int B, int Hkv, long long Tmax);
void alloc_carve(AllocParams& p, void* ws);
cudaError_t launch_allocate(AllocParams& p, cudaStream_t stream);
size_t retier_workspace_bytes(int B, int Hkv, long long Tmax, long long page_cap);
void retier_carve(AllocParams& p, void* ws);
// The allocation half of a re-tiering: tiers, row map, page table, headers
// of the rewritten pages and the released list (p.tier_out etc. are the
// store's own arrays; their old contents are snapshotted first).
cudaError_t launch_retier_plan(AllocParams& p, cudaStream_t stream);

// The data half: every row of a rewritten page, copied from its old row or,
// for a T0 row that becomes T1/T2, encoded from the fp16 K/V in its old page.
struct TranscodeParams {
  int B, Hkv;
  long long Tmax;
  int P;
  const int32_t* seq_lens;
  const uint8_t* tier;        // the new store
  const int32_t* row_of;
  const int32_t* indptr;
  const int32_t* tier_indptr;
  const uint32_t* ids;
  const int32_t* keep;        // [3U]
  long long page_cap;         // capacity of both page-id arrays
  const uint8_t* tier_old;    // the old store
  const int32_t* row_old;
  const int32_t* indptr_old;
  const uint32_t* ids_old;
  uint8_t* pool[3];
  long long slots[3];
  long long stride[3];
  int32_t* err;
  uint32_t* list;             // workspace: flat indices of the rows to write
  unsigned long long* count;  // workspace: their number
  float bx6[64], by6[64], bx4[16], by4[16];
  float bx5[32], by5[32];
  int t1_scheme;
  int share_grid;
};
cudaError_t launch_transcode(const TranscodeParams& p, cudaStream_t stream);
cudaError_t launch_dense_plan(AllocParams& p, cudaStream_t stream);

}  // namespace skv
