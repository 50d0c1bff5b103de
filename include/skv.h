/*
 * skv.h -- C-ABI of libskv: Spherical KV (Angle-Domain Attention + Rate-
 * Distortion Retention) paged decode on NVIDIA B200 (sm_100a).
 *
 * Sources: the pages about arXiv 2605.18856 "SPHERICAL KV: Angle-Domain
 * Attention and Rate-Distortion Retention for Efficient Long-Context
 * Inference": the gist.science technical summary, sections 1 (problem
 * statement), 2.1 (Angle-Domain Attention), 2.2 (Rate-Distortion Retention)
 * and 2.3 (system integration), and the arXiv abstract.
 *
 * Conventions (every entry point):
 *  - Returns an int status: SKV_OK or one of the SKV_ERR_* codes below.  On
 *    error, skv_last_error() gives a message (thread-local).  No C++
 *    exception crosses this boundary.
 *  - Device pointers are caller-owned device memory (the library never
 *    frees them).  Host pointers (config structs, pool descriptors) are read
 *    during the call only.
 *  - Every call that launches work takes a cudaStream_t (passed as void*,
 *    NULL = legacy default stream) and is asynchronous: it returns once the
 *    kernels are queued.  Errors found on the device are recorded in a
 *    caller-provided int32 device word (first error wins); skv_check()
 *    synchronises the stream, reads and clears it.
 *  - A context is bound to the CUDA device that was current at skv_create.
 *  - head_dim is 128 and the page size P is 16, 32 or 64 for the CUDA
 *    kernels.
 */
#ifndef SKV_H_
#define SKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define SKV_OK 0
#define SKV_ERR_ARG 1      /* invalid argument (host check or device check of an input)  */
#define SKV_ERR_BUDGET 2   /* protected tokens + page reserve exceed a sequence's budget  */
#define SKV_ERR_POOL 3     /* a free list or the page-id capacity is too short            */
#define SKV_ERR_CORRUPT 4  /* a page table entry or page header is out of range           */
#define SKV_ERR_CUDA 5     /* a CUDA runtime call failed                                   */
#define SKV_ERR_TIMEOUT 6  /* a bounded device-side wait ran out (kernel returned early)   */

/* tiers: T0 dense fp16 K/V, T1 6-bit angles, T2 4-bit angles, dropped */
#define SKV_TIER_T0 0
#define SKV_TIER_T1 1
#define SKV_TIER_T2 2
#define SKV_TIER_DROP 3

/* allocation modes */
#define SKV_MODE_QUOTA 0   /* fixed per-tier counts per (seq, head), ranked by utility */
#define SKV_MODE_BUDGET 1  /* rate-distortion greedy under a byte budget per sequence  */

/* query element types */
#define SKV_Q_FP16 0
#define SKV_Q_BF16 1

/* workspace kinds for skv_workspace_size */
#define SKV_WS_ALLOCATE 0
#define SKV_WS_DECODE 1
#define SKV_WS_DENSE_DECODE 2
#define SKV_WS_APPEND 3
#define SKV_WS_DECODE_UTILITY 4

/* host tables exported for tests (skv_tables) */
#define SKV_TABLE_BOUNDARY6_X 0  /* 64 fp32: cos((j+1/2) 2pi/64)                */
#define SKV_TABLE_BOUNDARY6_Y 1  /* 64 fp32: sin((j+1/2) 2pi/64)                */
#define SKV_TABLE_BOUNDARY4_X 2  /* 16 fp32                                      */
#define SKV_TABLE_BOUNDARY4_Y 3  /* 16 fp32                                      */
#define SKV_TABLE_KAPPA 4        /* 3 fp32: RDR slope per byte of each step      */
#define SKV_TABLE_RHO_LEVELS 5   /* 4 fp32: decoded share of each 2-bit code (the context's share grid) */
#define SKV_TABLE_BOUNDARY5_X 6  /* 32 fp32: cos((j+1/2) 2pi/32)                */
#define SKV_TABLE_BOUNDARY5_Y 7  /* 32 fp32: sin((j+1/2) 2pi/32)                */

typedef struct skv_config {
  int32_t head_dim;    /* d: 128 */
  int32_t page_size;   /* P: 16, 32 or 64 */
  int32_t outlier_protect; /* nonzero: skv_allocate also protects (keeps at T0)
                          every key with a pair whose share lies beyond twice
                          the share grid's top level, u = (rho/r) sqrt(d/2) > 4
                          (technical summary 2.2: outliers are among the
                          protected states) */
  int32_t t1_angle_bits; /* 0 or 6: T1 codes a pair as a 6-bit angle and a
                          2-bit share (levels u = 0.5, 1.0, 1.5, 2.0); 5: a 5-bit
                          angle and a 3-bit share (levels u = 0.25 .. 2.0 in
                          steps of 0.25), the same byte per pair.  The second
                          has about 40% lower logit error at the same 196 B */
  int32_t share_grid;  /* 0: the 2-bit share codes (T2, and T1 with 6 + 2 bits)
                          on the uniform levels u = 0.5, 1.0, 1.5, 2.0; 1: on
                          the exact Lloyd-Max grid of the Rayleigh density,
                          levels {383, 807, 1249, 1831} / 1024, thresholds
                          sqrt({22, 64, 145} / 64) (lower logit error at the
                          same bytes) */
  int32_t deterministic; /* nonzero: the decode never hands out pages at run
                          time (no dynamic chunks; see skv_decode_attention), so
                          repeated calls give bit-identical results; 0: the
                          unit-aligned split balances its runs' tails at run
                          time, and results may differ between calls in the
                          last bits (about 1e-5 relative) */
  int32_t t0_bf16;     /* nonzero: the fused T0 / bf16 path.  T0 rows hold K and V
                          as bf16 (each fp16 input rounded to nearest even, the
                          dense baseline's element type) and the decode takes
                          the dense kernel's bf16 logit and P.V path for T0
                          pages; needs the default T1 scheme and share grid.
                          skv_retier, which re-encodes T0 rows from their exact
                          fp16 keys, refuses such a store (SKV_ERR_ARG) */
  int32_t reserved[1]; /* zero */
} skv_config;

/* Device pools of page slots, one per tier.  Slot s of tier t starts at
   base[t] + s * stride(t) (skv_page_bytes); slots[t] is the slot count, used
   to bounds-check page ids on the device.  base[t] must be 128-byte aligned. */
typedef struct skv_pools {
  void* base[3];
  int64_t slots[3];
} skv_pools;

/* Device free lists: ids[t] holds len[t] slot numbers of tier t's pool, in
   the order in which they are handed out. */
typedef struct skv_free_lists {
  const uint32_t* ids[3];
  int64_t len[3];
} skv_free_lists;

typedef struct skv_ctx skv_ctx;

/* Create a context on the current CUDA device.  Computes the host tables
   (angle-sector boundaries, LUT cosines, share levels, RDR slopes) once.
   Errors: SKV_ERR_ARG for an unsupported head_dim / page_size. */
int skv_create(const skv_config* cfg, skv_ctx** out);

/* Destroy a context (NULL is accepted). */
int skv_destroy(skv_ctx* ctx);

/* Message of the last error on this thread ("" when none).  The pointer is
   valid until the next libskv call on this thread. */
const char* skv_last_error(void);

/* Page geometry of a tier (SPHERICAL KV technical summary 2.2: tier-
   homogeneous pages).  payload = 16 + P * bytes_per_token(tier); stride =
   payload rounded up to 128.  Bytes per (token, kv head): T0 512, T1 196,
   T2 180.  tier SKV_TIER_DROP + 1 (= 4) asks for the dense-bf16 baseline
   page (same as T0). */
int skv_page_bytes(const skv_ctx* ctx, int tier, int64_t* payload, int64_t* stride);

/* Copy host table `which` (SKV_TABLE_*) into out[0..n).  Host memory. */
int skv_tables(const skv_ctx* ctx, int which, float* out, int64_t n);

/* Number of SMs of the context's device and the default split count that
   skv_decode_attention uses when num_splits == 0. */
int skv_device_info(const skv_ctx* ctx, int* sm_count, int* default_splits);

/* Bytes of device workspace that a call needs.
   SKV_WS_ALLOCATE: skv_allocate on B sequences x Hkv heads x Tmax tokens.
   SKV_WS_APPEND: skv_append on B x Hkv units; Tmax carries the page-id
   capacity (page_cap) instead.
   SKV_WS_DECODE / SKV_WS_DENSE_DECODE: the decode with num_splits chunks
   (0 = default) over B x Hkv units with Hq query heads.
   SKV_WS_DECODE_UTILITY: skv_decode_utility; Tmax carries the page-id
   capacity (page_cap): the decode's scratch plus page_cap * P * (Hq/Hkv)
   fp32 captured logits.  The workspace is
   scratch that the call may overwrite; it must stay allocated until the
   stream has run the call. */
int skv_workspace_size(const skv_ctx* ctx, int which, int B, int Hkv, int Hq, int64_t Tmax,
                       int num_splits, size_t* bytes);

/* skv_allocate -- Rate-Distortion Retention (technical summary 2.2; abstract:
   "keep/drop decisions and precision tiers per token and head under a fixed
   budget, producing tier-homogeneous pages with lightweight metadata").
   Chooses a tier for every (seq b, kv head h, position t < seq_lens[b]),
   packs the kept tokens into tier-homogeneous pages and writes the page
   table and page headers.
     K          fp16 [B][Hkv][Tmax][128] device: keys (radius from exact norm)
     seq_lens   int32 [B] device, 0 <= seq_lens[b] <= Tmax
     utility    fp32 [B][Hkv][Tmax] device, finite and >= 0 (budget mode
                required; quota mode: NULL ranks by position)
     protect    uint8 [B][Hkv][Tmax] device or NULL: nonzero = always T0
     mode       SKV_MODE_BUDGET: the greedy rate-distortion walk under
                budget[b] bytes per sequence (shared by its Hkv heads).
                SKV_MODE_QUOTA: per (b, h) the quota[b][0..2] highest-utility
                unprotected tokens go to T0, T1, T2 in that order.
     budget     int64 [B] device (budget mode) or NULL
     quota      int32 [B][3] device (quota mode) or NULL
     free       per-tier free lists (device ids, host descriptor)
     pools      per-tier pools; headers are written into each used slot and
                every row of a partial page is zeroed
     tier_out   uint8 [B][Hkv][Tmax] device: 0 T0, 1 T1, 2 T2, 3 dropped
                (positions >= seq_lens[b] are 3)
     row_of     int32 [B][Hkv][Tmax] device: page index within the unit's
                list * P + row, or -1 when not resident
     page_indptr int32 [B*Hkv + 1] device: CSR offsets per unit b*Hkv + h
     page_tier_indptr int32 [3*B*Hkv + 1] device or NULL: CSR offsets per
                (unit, tier) segment 3*u + t (entry 3u = page_indptr[u]);
                lets the decode split its work by streamed bytes
     page_ids   uint32 [page_cap] device: tier << 30 | slot; per unit the T0
                pages, then T1, then T2
     err_word   int32 device: SKV_ERR_BUDGET, SKV_ERR_POOL or SKV_ERR_ARG
                found on the device (outputs are then unspecified)
     workspace  device scratch of skv_workspace_size(SKV_WS_ALLOCATE) bytes */
int skv_allocate(skv_ctx* ctx, const uint16_t* K, int B, int Hkv, int64_t Tmax,
                 const int32_t* seq_lens, const float* utility, const uint8_t* protect,
                 int mode, const int64_t* budget, const int32_t* quota,
                 const skv_free_lists* free, const skv_pools* pools, uint8_t* tier_out,
                 int32_t* row_of, int32_t* page_indptr, int32_t* page_tier_indptr,
                 uint32_t* page_ids, int64_t page_cap, int32_t* err_word, void* workspace,
                 size_t ws_bytes, void* stream);

/* skv_encode -- maps dense keys to spherical codes (technical summary 2.1,
   2.3): for every resident (b, h, t) writes its row of the page that
   row_of / page_indptr / page_ids assign:
     T0: fp16 K and V unchanged (in the documented within-page order)
     T1/T2: r~ = fp16 |k|, per pair a 6-bit (T1) or 4-bit (T2) angle code and
            a 2-bit share code, int8 V with a per-token fp16 absmax scale.
   Arguments as for skv_allocate (tier/row_of/page table are its outputs).
   Page ids are bounds-checked (SKV_ERR_CORRUPT). */
int skv_encode(skv_ctx* ctx, const uint16_t* K, const uint16_t* V, int B, int Hkv, int64_t Tmax,
               const int32_t* seq_lens, const uint8_t* tier, const int32_t* row_of,
               const int32_t* page_indptr, const uint32_t* page_ids, const skv_pools* pools,
               int32_t* err_word, void* stream);

/* skv_append -- decode-time ingest of the newest token (technical summary
   2.2: protected tokens keep the top tier; 2.3 / abstract: the paged store
   of the serving loop).  The paper states no per-step update of the store;
   this is the plainest one: the token at position t = seq_lens[b] of every
   kv head h becomes resident as T0 (the newest token lies in the protected
   recent window).  It takes the next row of its unit's last T0 page, or,
   when that page is full or the unit has no T0 page, a new T0 page whose
   slot is free0[*free0_cursor + k] (k counts the units that need one, in
   unit order) inserted at the end of the unit's T0 segment; later page ids
   move up and the unit's T1/T2 rows move one page down in row_of.  The
   store then equals what skv_allocate + skv_encode give for the same tiers
   (page slots aside).  skv_retier later demotes the rows that leave the
   protected window.
     K_new, V_new  fp16 [B][Hkv][128] device: the new token's key and value
     Tmax          capacity of tier/row_of; seq_lens[b] < Tmax is required
     seq_lens      int32 [B] device, incremented by one
     tier, row_of, page_indptr, page_tier_indptr (required), page_ids: the
                   store's arrays as skv_allocate wrote them, updated
     page_cap      capacity of page_ids
     pools         the pools (only the T0 pool is written)
     free0, free0_len  T0 free slots (device); *free0_cursor (device int32)
                   is the first unused entry and is advanced
     workspace     skv_workspace_size(SKV_WS_APPEND, B, Hkv, 0, page_cap) bytes
   Device errors: SKV_ERR_ARG (seq_lens[b] >= Tmax), SKV_ERR_POOL (free list
   or page capacity exhausted), SKV_ERR_CORRUPT (bad last T0 page id); the
   store is then left unchanged. */
int skv_append(skv_ctx* ctx, const uint16_t* K_new, const uint16_t* V_new, int B, int Hkv,
               int64_t Tmax, int32_t* seq_lens, uint8_t* tier, int32_t* row_of,
               int32_t* page_indptr, int32_t* page_tier_indptr, uint32_t* page_ids,
               int64_t page_cap, const skv_pools* pools, const uint32_t* free0,
               int64_t free0_len, int32_t* free0_cursor, int32_t* err_word, void* workspace,
               size_t ws_bytes, void* stream);

/* skv_retier -- re-tiering of rows leaving the protected recent window, on
   the store itself (technical summary 2.2, Rate-Distortion Retention: keep
   or drop and the tier are per-token, per-head decisions under a fixed
   budget; 2.3, System Integration: the retention filter sits between the
   codes and the paged store).  The demoted rows are T0 rows; their exact
   fp16 K and V are read back from their T0 pages, so no dense K/V is
   needed.  Every other resident token keeps its tier.  The demoted rows are
   re-decided by the budget walk of skv_allocate: with
     left = budget[b] - (bytes of the kept tokens) - Hkv (P-1) (512+196+180)
   their upgrade steps (drop->T2, T2->T1, T1->T0; keys u fp32(r^2) kappa,
   ties by step, head, position) are taken in order while they fit, so a
   demoted row ends T0, T1, T2 or dropped.  The store is then what
   skv_allocate's layout + skv_encode give for the new tiers (page slots
   aside), updated in place: in each (unit, tier) page segment the pages
   wholly before the first changed row keep their slots; the later pages
   are rewritten into slots free->ids[t][free_cursor[t] + k] and the old ones
   are listed in `released`.
     seq_lens      int32 [B] device (unchanged)
     utility       fp32 [B][Hkv][Tmax] device: utilities of the demoted rows
     demote        uint8 [B][Hkv][Tmax] device: 1 = re-decide this row (it must
                   be resident T0; SKV_ERR_ARG otherwise, the row then kept)
     budget        int64 [B] device: bytes per sequence
     free, free_cursor  device free lists per tier and int32 [3] device
                   cursors (first unused entry), advanced by the slots taken
     pools         the pools of the store (128-byte aligned)
     tier, row_of, page_indptr, page_tier_indptr (required), page_ids: the
                   store's arrays, rewritten
     page_cap      capacity of page_ids
     released      uint32 [page_cap] device: ids (tier << 30 | slot) of the old
                   pages that the store no longer references; n_released
                   (int32 device) their count.  They may go back to the
                   caller's free lists once the call has completed.
     workspace     skv_retier_workspace_size() bytes of device scratch
   Device errors: SKV_ERR_BUDGET when the kept tokens and the reserve
   exceed a sequence's budget (its demoted rows are then dropped; the store
   stays consistent); SKV_ERR_POOL (free list or page capacity exhausted)
   and SKV_ERR_CORRUPT (a bad page id or row) leave the store invalid: it
   must be rebuilt with skv_allocate + skv_encode.  B * Hkv * Tmax must be
   below 2^32 (SKV_ERR_ARG otherwise).  Budget mode only; no
   outlier protection is applied to the demoted rows (leave such rows out of
   `demote`). */
int skv_retier_workspace_size(const skv_ctx* ctx, int B, int Hkv, int64_t Tmax,
                              int64_t page_cap, size_t* bytes);
int skv_retier(skv_ctx* ctx, int B, int Hkv, int64_t Tmax, const int32_t* seq_lens,
               const float* utility, const uint8_t* demote, const int64_t* budget,
               const skv_free_lists* free, int32_t* free_cursor, const skv_pools* pools,
               uint8_t* tier, int32_t* row_of, int32_t* page_indptr,
               int32_t* page_tier_indptr, uint32_t* page_ids, int64_t page_cap,
               uint32_t* released, int32_t* n_released, int32_t* err_word, void* workspace,
               size_t ws_bytes, void* stream);

/* skv_decode_attention -- the ADA decode step (technical summary 2.1: logits
   computed directly from the radius and angle codes, no dense key
   materialised; abstract: "paged, block-local, fusion-friendly decode path").
   For every sequence b and query head hq (kv head h = hq / (Hq/Hkv)):
     out[b][hq] = sum_t softmax_t(l_t) v^_t,  lse[b][hq] = log sum_t exp(l_t)
   over the resident tokens of (b, h): l_t = (r~_t/sqrt d) sum_i rho^_i
   LUT_i[c_i] for T1/T2 (LUT_i[c] = q_{2i} cos(2 pi c/2^b) + q_{2i+1}
   sin(2 pi c/2^b)), q . k_t / sqrt d for T0; v^ = scale * int8 or fp16 V.
     q        [B][Hq][128] device, q_dtype SKV_Q_BF16 or SKV_Q_FP16
     Hq       a multiple of Hkv with Hq/Hkv in {1, 2, 4}
     page_indptr / page_ids / pools: the paged store (any slots, any order of
              pages within a unit; pages are streamed whole)
     page_tier_indptr  NULL, or skv_allocate's per-(unit, tier) offsets: the
              runs are then cut by payload bytes instead of page counts
              (same results either way).  When num_splits >= 8*B*Hkv
              every unit gets its own runs, in proportion to its cost, and
              about the last eighth of a unit's pages (whole chunks of 512
              tokens) is handed out at run time, chunk by chunk, to the
              unit's runs as they finish their static part (unless the
              context is deterministic); otherwise the
              page list of all units is cut into runs of equal cost.
     out      fp32 [B][Hq][128] device; lse fp32 [B][Hq] device or NULL
              (a unit without resident tokens gives out 0, lse -inf)
     num_splits  number of page runs = CTAs (0 = default: the SM count)
     workspace   skv_workspace_size(SKV_WS_DECODE, ..., num_splits) bytes;
              its contents need no initialisation (the chunk counters carry
              a per-launch tag and are reset by the launch that uses them),
              but two decodes that overlap in time must not share one
   Stream order: the decode is launched as a programmatic dependent of the
   stream's previous kernel.  If that kernel lets its dependents start
   early (griddepcontrol.launch_dependents, as this library's merge and
   utility kernels do), the decode may read the page table and the pages
   before that kernel has finished; it reads q and writes out, lse and
   the workspace only after it has (a corrupt page id may be reported into
   err_word, atomically, before).  So a kernel that writes the
   store must not let its dependents start early (none in this library
   does); q and the outputs follow ordinary stream order.
   Device errors: SKV_ERR_CORRUPT (bad page id / header: the page is
   skipped), SKV_ERR_TIMEOUT (a bounded wait ran out). */
int skv_decode_attention(skv_ctx* ctx, const void* q, int q_dtype, int B, int Hq, int Hkv,
                         const int32_t* page_indptr, const int32_t* page_tier_indptr,
                         const uint32_t* page_ids, const skv_pools* pools, float* out, float* lse, int32_t* err_word,
                         void* workspace, size_t ws_bytes, int num_splits, void* stream);

/* skv_decode_attention_host -- one decode step from and to host memory
   (an interface convenience of this library; the operation is that of
   skv_decode_attention): copies q_host to q_dev, runs the decode, copies
   out and lse back to out_host / lse_host, synchronises the stream and
   returns the device error word's verdict as skv_check does (and resets
   it).  Every copy is a single cudaMemcpyAsync on `stream`; use pinned
   host buffers so that they are asynchronous DMA transfers.  With lse_dev
   and lse_host both NULL, lse lives right after out in the same buffers
   (out_dev / out_host then hold B*Hq*129 floats: out, then lse) and one
   copy returns both.  A stream other than the legacy default stream saves
   the default stream's implicit synchronisation (about 4 us a step).
     q_host    [B][Hq][128] 16-bit host buffer (q_dtype as for the decode)
     q_dev     device buffer of the same size (caller-owned scratch)
     out_dev / lse_dev   device fp32 [B][Hq][128] / [B][Hq] scratch
     out_host / lse_host host fp32 [B][Hq][128] / [B][Hq] results
     other arguments as for skv_decode_attention (lse is required here)
   Returns SKV_OK, an argument / CUDA error, or the device error the step
   reported (SKV_ERR_CORRUPT, SKV_ERR_TIMEOUT).  Blocks the calling thread
   until the step is done.  The context holds one pinned word for the error
   copy: calls on one context from several host threads must not overlap. */
int skv_decode_attention_host(skv_ctx* ctx, const void* q_host, int q_dtype, int B, int Hq,
                              int Hkv, const int32_t* page_indptr,
                              const int32_t* page_tier_indptr, const uint32_t* page_ids,
                              const skv_pools* pools, void* q_dev, float* out_dev, float* lse_dev,
                              float* out_host, float* lse_host, int32_t* err_word,
                              void* workspace, size_t ws_bytes, int num_splits, void* stream);

/* skv_decode_attention_host_pipelined -- the host step of
   skv_decode_attention_host, pipelined across calls so that one step's
   copies and the host's wait overlap the next step's decode.  Call k issues
   step k: q_host -> slot k%2 of q_dev on a copy stream of the context, the
   decode on `stream` once that copy is done, then out and lse packed into
   res_host (B*Hq*128 floats of out, then B*Hq of lse) and the step's error
   word on a second copy stream of the context once the decode is done.  It
   returns once step k-1 is done: step k-1's results are then in the
   res_host given to call k-1, and the return value is step k-1's status
   (SKV_OK for the first call).  The caller therefore alternates two sets of
   host buffers (q_host, res_host): the set of call k must not be touched
   until call k+1 has returned.  skv_decode_attention_host_drain waits for
   the last step issued and returns its status; call it before the buffers
   are used otherwise, before the stream changes and before skv_destroy.
     q_dev      device scratch of 2 x B*Hq*128 16-bit values (two slots)
     res_dev    device scratch of 2 x B*Hq*129 floats (two slots)
     other arguments as for skv_decode_attention_host (the error words are
     the context's own)
   Calls on one context must not overlap. */
int skv_decode_attention_host_pipelined(skv_ctx* ctx, const void* q_host, int q_dtype, int B,
                                        int Hq, int Hkv, const int32_t* page_indptr,
                                        const int32_t* page_tier_indptr,
                                        const uint32_t* page_ids, const skv_pools* pools,
                                        void* q_dev, float* res_dev, float* res_host,
                                        void* workspace, size_t ws_bytes, int num_splits,
                                        void* stream);
int skv_decode_attention_host_drain(skv_ctx* ctx);

/* skv_merge_partials -- the exchange step of a context-parallel decode.
   Each of R ranks attends (skv_decode_attention) over its own slice of every
   sequence's tokens; softmax over the union of disjoint slices factors into
   the slices' normalised outputs weighted by their denominators:
     M = max_r lse_r,  w_r = exp(lse_r - M),
     out = sum_r w_r out_r / sum_r w_r,   lse = M + log sum_r w_r
   (partials with lse = -inf carry no weight; all empty gives out 0 and lse
   -inf, as the decode gives for an empty unit).  The pages fix attention over
   all resident tokens (technical summary 2.1); splitting it by slices is
   this library's multi-GPU layout, not the paper's.
     n            rows (B * Hq)
     out_parts    fp32 device, rank r's out [n][128] at out_parts + r*rank_stride
     lse_parts    fp32 device, rank r's lse [n] at lse_parts + r*rank_stride
     rank_stride  floats between ranks (both arrays); e.g. a packed all-gather
                  buffer of R blocks {out [n][128], lse [n], one pad float when
                  n is odd} has out_parts = buf, lse_parts = buf + 128 n,
                  rank_stride = 129 n + (n & 1)
     out, lse     fp32 device [n][128] and [n] (lse may be NULL)
   out_parts, out and rank_stride must be 8-byte aligned (float2 loads). */
int skv_merge_partials(skv_ctx* ctx, int R, int64_t n, const float* out_parts,
                       const float* lse_parts, int64_t rank_stride, float* out, float* lse,
                       void* stream);

/* skv_decode_utility -- the decode of skv_decode_attention plus the
   utility update that closes the retention loop.  The abstract's retention
   decides by "estimated future utility" without saying how it is estimated;
   this library's reading is the attention mass the decode itself computes:
     mass[b][h][t] = sum_{g < G} softmax_t(l_{hG+g})[t]   (0 if dropped)
     utility[b][h][t] <- gamma * utility[b][h][t] + mass[b][h][t]
   for every t < seq_lens[b] (positions past it are left unchanged), so that
   gamma = 1 keeps the running sum and gamma < 1 a geometric decay.  The
   decode stores each resident row's logit (fp32, log2 domain) in the
   workspace as it streams the pages; a second kernel forms the mass from
   those logits and the merged lse.  The result feeds skv_allocate's utility.
     q ... num_splits   as for skv_decode_attention (lse is required)
     page_cap      capacity of page_ids (rows of the logit scratch / P)
     Tmax, seq_lens, tier, row_of   skv_allocate's / skv_append's outputs
                   for the same store (device; row_of locates a token's row)
     gamma         decay of the previous utility (host float)
     utility       fp32 [B][Hkv][Tmax] device, updated in place
     workspace     skv_workspace_size(SKV_WS_DECODE_UTILITY, B, Hkv, Hq,
                   page_cap, num_splits) bytes
   Device errors: as skv_decode_attention, plus SKV_ERR_CORRUPT when a
   resident token's row lies outside its unit's pages (its utility is then
   left unchanged) and SKV_ERR_ARG when page_cap is below the page count. */
int skv_decode_utility(skv_ctx* ctx, const void* q, int q_dtype, int B, int Hq, int Hkv,
                       const int32_t* page_indptr, const int32_t* page_tier_indptr,
                       const uint32_t* page_ids, int64_t page_cap, const skv_pools* pools,
                       int64_t Tmax, const int32_t* seq_lens, const uint8_t* tier,
                       const int32_t* row_of, float gamma, float* utility, float* out, float* lse,
                       int32_t* err_word, void* workspace, size_t ws_bytes, int num_splits,
                       void* stream);

/* skv_decode_attention_static -- skv_decode_attention without a caller
   workspace (the paper has no counterpart: this is an interface convenience
   of this library).  Same arguments, results and device errors as
   skv_decode_attention (ADA decode only; page_tier_indptr may be NULL), but
   the split partials and run ranges live in a fixed 4 MiB device
   array inside libskv, so the call allocates nothing.
     - A call that would need more than 4 MiB of scratch (the size
       skv_workspace_size(SKV_WS_DECODE) reports) is refused with
       SKV_ERR_ARG before anything is launched.
     - The array is shared by every call on a device: calls that overlap in
       time (on different streams or host threads) race on it.  Serialise
       them, e.g. by issuing them on one stream.
     - The first call on each device looks up the array's device address and
       configures the kernel; make it before any stream capture begins on
       that device. */
int skv_decode_attention_static(skv_ctx* ctx, const void* q, int q_dtype, int B, int Hq,
                                int Hkv, const int32_t* page_indptr,
                                const int32_t* page_tier_indptr, const uint32_t* page_ids,
                                const skv_pools* pools, float* out, float* lse,
                                int32_t* err_word, int num_splits, void* stream);

/* skv_dense_pack_bf16 -- the dense baseline's store: every token of every
   (b, h) kept as bf16 K/V (fp16 inputs rounded to nearest even) in pages of
   P rows with the T0 page layout.  Slots come from free_ids in (b, h, page)
   order.  Writes page_indptr [B*Hkv+1] and page_ids (tier bits 0). */
int skv_dense_pack_bf16(skv_ctx* ctx, const uint16_t* K, const uint16_t* V, int B, int Hkv,
                        int64_t Tmax, const int32_t* seq_lens, const uint32_t* free_ids,
                        int64_t free_len, void* pool, int64_t pool_slots, int32_t* page_indptr,
                        uint32_t* page_ids, int64_t page_cap, int32_t* err_word,
                        void* workspace, size_t ws_bytes, void* stream);

/* skv_dense_decode_bf16 -- dense bf16 paged-decode baseline: textbook
   attention over every token of the bf16 pages, the same kernel skeleton as
   skv_decode_attention (split-K, GQA, online softmax, P.V on tensor cores). */
int skv_dense_decode_bf16(skv_ctx* ctx, const void* q, int q_dtype, int B, int Hq, int Hkv,
                          const int32_t* page_indptr, const uint32_t* page_ids,
                          const void* pool, int64_t pool_slots, float* out, float* lse,
                          int32_t* err_word, void* workspace, size_t ws_bytes, int num_splits,
                          void* stream);

/* Profiling aid: when `event` (a cudaEvent_t, or NULL to clear) is set, every
   later skv_decode_attention / skv_dense_decode_bf16 call on this context
   records it on its stream between the decode kernel and the merge kernel,
   so that a caller can time the decode kernel alone with CUDA events. */
int skv_set_profile_event(skv_ctx* ctx, void* event);

/* The decode's bounded waits (the planner, issuers and consumers of a CTA
   wait on shared-memory barriers for one another and for page copies): a
   wait that runs longer than `cycles` SM clocks ends the CTA's work and
   reports SKV_ERR_TIMEOUT in err_word; later calls work normally.  0 (the
   default) means about one second.  A short limit exists to exercise that
   error path: before the CTA leaves, every page copy it started is waited
   for with the one-second limit, whatever `cycles` is. */
int skv_set_wait_limit(skv_ctx* ctx, int64_t cycles);

/* Synchronise `stream`, read the device error word, reset it to 0 and return
   SKV_OK or the recorded SKV_ERR_* code. */
int skv_check(skv_ctx* ctx, int32_t* err_word, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SKV_H_ */
