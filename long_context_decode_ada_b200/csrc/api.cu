// api.cu -- the extern "C" entry points of libskv (declared in include/skv.h).
// Host-side argument checks, the context's constant tables and the kernel
// launches.  No allocation happens here except the context struct itself.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/skv.h"
#include "common.cuh"
#include "kernels.h"

struct skv_ctx {
  int d;
  int P;
  int log2P;
  int device;
  int sm_count;
  size_t smem_optin;
  float bx6[64], by6[64], bx4[16], by4[16], bx5[32], by5[32];
  float cos6[64], sin6[64], cos4[16], sin4[16], cos5[32], sin5[32];
  int t1_scheme = 0;            // 0: 6-bit angle + 2-bit share; 1: 5-bit + 3-bit
  int share_grid = 0;           // 2-bit share grid: 0 uniform, 1 Lloyd-Max
  int deterministic = 0;        // the decode's split is static (no run-time chunks)
  int t0_bf16 = 0;              // T0 rows in bf16, decoded on the bf16 path
  long long wait_limit = 0;     // decode waits: SM clocks (0: the default, about 1 s)
  float kappa[3];
  float rho_levels[4];
  long long payload[4];
  long long stride[4];
  cudaEvent_t profile_event;
  int32_t* err_host = nullptr;  // pinned word for skv_decode_attention_host (lazily allocated)
  int outlier_protect = 0;      // skv_config.outlier_protect
  // skv_decode_attention_host_pipelined: per slot (two steps in flight) a
  // device and a pinned error word and the events of the q copy, the decode
  // and the result copies; the copy streams; the steps issued
  int32_t* pipe_err = nullptr;       // pinned [2]
  int32_t* pipe_err_dev = nullptr;   // device [2]
  cudaEvent_t pipe_ev_q[2] = {nullptr, nullptr};
  cudaEvent_t pipe_ev_d[2] = {nullptr, nullptr};
  cudaEvent_t pipe_ev_r[2] = {nullptr, nullptr};
  cudaStream_t pipe_in = nullptr, pipe_out = nullptr;
  long long pipe_n = 0;
  bool pipe_pending = false;
  void* pipe_stream = nullptr;
};

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int ok() {
  g_err.clear();
  return SKV_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(SKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Relative mean-squared logit error of a b-bit uniform angle quantiser:
// 2 (1 - sin(x)/x), x = pi / 2^b (half the sector width).
double angle_distortion(int b) {
  const double x = M_PI / (double)(1 << b);
  return 2.0 * (1.0 - std::sin(x) / x);
}

bool valid_pools(const skv_pools* pools, int ntiers) {
  if (!pools) return false;
  for (int t = 0; t < ntiers; ++t) {
    if (pools->slots[t] < 0) return false;
    if (pools->slots[t] > 0 && !pools->base[t]) return false;
    if ((reinterpret_cast<uintptr_t>(pools->base[t]) & 127) != 0) return false;
  }
  return true;
}

}  // namespace

// ---------------------------------------------------------------------------
// Fixed decode scratch for skv_decode_attention_static: the split partials
// and the units' run ranges live in this array instead of a caller
// workspace.  Its device address is looked up once per device.
// ---------------------------------------------------------------------------
constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

static std::mutex g_scratch_mu;
static void* g_scratch_ptr[64] = {};

// The scratch's device address on the current device (looked up once per
// device, with that device current).  Returns the CUDA status.
static cudaError_t static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

extern "C" {

const char* skv_last_error(void) { return g_err.c_str(); }

int skv_create(const skv_config* cfg, skv_ctx** out) {
  if (!cfg || !out) return fail(SKV_ERR_ARG, "skv_create: null argument");
  *out = nullptr;
  if (cfg->head_dim != 128) return fail(SKV_ERR_ARG, "head_dim must be 128 (got %d)", cfg->head_dim);
  const int P = cfg->page_size;
  if (P != 16 && P != 32 && P != 64) return fail(SKV_ERR_ARG, "page_size must be 16, 32 or 64");
  skv_ctx* c = new (std::nothrow) skv_ctx();
  if (!c) return fail(SKV_ERR_ARG, "out of host memory");
  c->d = 128;
  c->P = P;
  c->outlier_protect = cfg->outlier_protect != 0;
  if (cfg->t1_angle_bits != 0 && cfg->t1_angle_bits != 5 && cfg->t1_angle_bits != 6) {
    delete c;
    return fail(SKV_ERR_ARG, "t1_angle_bits must be 0, 5 or 6 (got %d)", cfg->t1_angle_bits);
  }
  c->t1_scheme = cfg->t1_angle_bits == 5;
  if (cfg->share_grid != 0 && cfg->share_grid != 1) {
    delete c;
    return fail(SKV_ERR_ARG, "share_grid must be 0 or 1 (got %d)", cfg->share_grid);
  }
  c->share_grid = cfg->share_grid;
  c->deterministic = cfg->deterministic != 0;
  c->t0_bf16 = cfg->t0_bf16 != 0;
  if (c->t0_bf16 && (c->t1_scheme || c->share_grid)) {
    delete c;
    return fail(SKV_ERR_ARG, "t0_bf16 needs the default T1 scheme and share grid");
  }
  c->log2P = P == 16 ? 4 : (P == 32 ? 5 : 6);
  c->device = 0;
  c->profile_event = nullptr;
  c->sm_count = 148;
  c->smem_optin = 232448;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    c->device = dev;
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
      c->sm_count = v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess &&
        v > 0)
      c->smem_optin = (size_t)v;
  } else {
    cudaGetLastError();
  }
  for (int j = 0; j < 64; ++j) {
    const double beta = (j + 0.5) * (2.0 * M_PI / 64.0);
    c->bx6[j] = (float)std::cos(beta);
    c->by6[j] = (float)std::sin(beta);
    const double a = 2.0 * M_PI * j / 64.0;
    c->cos6[j] = (float)std::cos(a);
    c->sin6[j] = (float)std::sin(a);
  }
  for (int j = 0; j < 32; ++j) {
    const double beta = (j + 0.5) * (2.0 * M_PI / 32.0);
    c->bx5[j] = (float)std::cos(beta);
    c->by5[j] = (float)std::sin(beta);
    const double a = 2.0 * M_PI * j / 32.0;
    c->cos5[j] = (float)std::cos(a);
    c->sin5[j] = (float)std::sin(a);
  }
  for (int j = 0; j < 16; ++j) {
    const double beta = (j + 0.5) * (2.0 * M_PI / 16.0);
    c->bx4[j] = (float)std::cos(beta);
    c->by4[j] = (float)std::sin(beta);
    const double a = 2.0 * M_PI * j / 16.0;
    c->cos4[j] = (float)std::cos(a);
    c->sin4[j] = (float)std::sin(a);
  }
  const double c6 = angle_distortion(6), c4 = angle_distortion(4);
  c->kappa[0] = (float)((1.0 - c4) / 180.0);
  c->kappa[1] = (float)((c4 - c6) / 16.0);
  c->kappa[2] = (float)(c6 / 316.0);
  // decoded share of each 2-bit code: u_s / sqrt(d/2) on the context's grid
  static const double kLevelsLM[4] = {383.0 / 1024, 807.0 / 1024, 1249.0 / 1024, 1831.0 / 1024};
  for (int k = 0; k < 4; ++k)
    c->rho_levels[k] = (float)(c->share_grid ? kLevelsLM[k] / 8.0 : (k + 1) / 16.0);
  const int rowb[4] = {512, 196, 180, 512};
  for (int t = 0; t < 4; ++t) {
    c->payload[t] = skv::kHdrBytes + (long long)P * rowb[t];
    c->stride[t] = (c->payload[t] + 127) / 128 * 128;
  }
  *out = c;
  return ok();
}

int skv_destroy(skv_ctx* ctx) {
  if (ctx && ctx->err_host) cudaFreeHost(ctx->err_host);
  if (ctx && ctx->pipe_err) cudaFreeHost(ctx->pipe_err);
  if (ctx && ctx->pipe_err_dev) cudaFree(ctx->pipe_err_dev);
  for (int i = 0; ctx && i < 2; ++i) {
    if (ctx->pipe_ev_q[i]) cudaEventDestroy(ctx->pipe_ev_q[i]);
    if (ctx->pipe_ev_d[i]) cudaEventDestroy(ctx->pipe_ev_d[i]);
    if (ctx->pipe_ev_r[i]) cudaEventDestroy(ctx->pipe_ev_r[i]);
  }
  if (ctx && ctx->pipe_in) cudaStreamDestroy(ctx->pipe_in);
  if (ctx && ctx->pipe_out) cudaStreamDestroy(ctx->pipe_out);
  delete ctx;
  return ok();
}

int skv_page_bytes(const skv_ctx* ctx, int tier, int64_t* payload, int64_t* stride) {
  if (!ctx || tier < 0 || tier > 4 || tier == SKV_TIER_DROP)
    return fail(SKV_ERR_ARG, "skv_page_bytes: bad tier %d", tier);
  const int t = tier == 4 ? 3 : tier;
  if (payload) *payload = ctx->payload[t];
  if (stride) *stride = ctx->stride[t];
  return ok();
}

int skv_tables(const skv_ctx* ctx, int which, float* out, int64_t n) {
  if (!ctx || !out) return fail(SKV_ERR_ARG, "skv_tables: null argument");
  const float* src = nullptr;
  int64_t len = 0;
  switch (which) {
    case SKV_TABLE_BOUNDARY6_X: src = ctx->bx6; len = 64; break;
    case SKV_TABLE_BOUNDARY6_Y: src = ctx->by6; len = 64; break;
    case SKV_TABLE_BOUNDARY4_X: src = ctx->bx4; len = 16; break;
    case SKV_TABLE_BOUNDARY4_Y: src = ctx->by4; len = 16; break;
    case SKV_TABLE_KAPPA: src = ctx->kappa; len = 3; break;
    case SKV_TABLE_RHO_LEVELS: src = ctx->rho_levels; len = 4; break;
    case SKV_TABLE_BOUNDARY5_X: src = ctx->bx5; len = 32; break;
    case SKV_TABLE_BOUNDARY5_Y: src = ctx->by5; len = 32; break;
    default: return fail(SKV_ERR_ARG, "skv_tables: unknown table %d", which);
  }
  if (n < len) return fail(SKV_ERR_ARG, "skv_tables: need %lld floats", (long long)len);
  std::memcpy(out, src, sizeof(float) * len);
  return ok();
}

int skv_device_info(const skv_ctx* ctx, int* sm_count, int* default_splits) {
  if (!ctx) return fail(SKV_ERR_ARG, "skv_device_info: null ctx");
  if (sm_count) *sm_count = ctx->sm_count;
  if (default_splits) *default_splits = ctx->sm_count;
  return ok();
}

// The decode's split weight of one page of tier ti (3: a dense bf16 page):
// its payload bytes, a T2 page at least a T1 page's (their rows take about
// the same consumer time), a T0 page SKV_T0_COST_PCT percent of its bytes.
#ifndef SKV_T0_COST_PCT
#define SKV_T0_COST_PCT 100
#endif
static long long split_cost(const skv_ctx* ctx, int ti) {
  if (ti == 3) return ctx->payload[3];
  if (ti == 0) return ctx->payload[0] * SKV_T0_COST_PCT / 100;
  if (ti == 1) return ctx->payload[1];
  return std::max(ctx->payload[2], ctx->payload[1]);
}

static int decode_splits(const skv_ctx* ctx, int num_splits) {
  return num_splits > 0 ? num_splits : ctx->sm_count;
}

// offset of the logit rows in a SKV_WS_DECODE_UTILITY workspace (256-byte aligned)
static size_t decode_utility_logits_at(long long S, long long U, int G) {
  return (skv::decode_ws(S, U, G).bytes + 255) / 256 * 256;
}

int skv_workspace_size(const skv_ctx* ctx, int which, int B, int Hkv, int Hq, int64_t Tmax,
                       int num_splits, size_t* bytes) {
  if (!ctx || !bytes) return fail(SKV_ERR_ARG, "skv_workspace_size: null argument");
  if (B < 0 || Hkv <= 0 || Tmax < 0) return fail(SKV_ERR_ARG, "skv_workspace_size: bad sizes");
  if (which == SKV_WS_ALLOCATE) {
    *bytes = skv::alloc_workspace_bytes(B, Hkv, Tmax);
    return ok();
  }
  if (which == SKV_WS_DECODE || which == SKV_WS_DENSE_DECODE) {
    if (Hq <= 0 || Hq % Hkv != 0) return fail(SKV_ERR_ARG, "Hq must be a multiple of Hkv");
    const int G = Hq / Hkv;
    const long long S = decode_splits(ctx, num_splits);
    // split partials, then each unit's range of runs
    *bytes = skv::decode_ws(S, (long long)B * Hkv, G).bytes;
    return ok();
  }
  if (which == SKV_WS_DECODE_UTILITY) {
    // Tmax carries the page-id capacity here: the decode's scratch, then the
    // captured logits of page_cap * P rows x G heads
    if (Hq <= 0 || Hq % Hkv != 0) return fail(SKV_ERR_ARG, "Hq must be a multiple of Hkv");
    const int G = Hq / Hkv;
    const long long S = decode_splits(ctx, num_splits);
    *bytes = decode_utility_logits_at(S, (long long)B * Hkv, G) +
             (size_t)Tmax * (size_t)ctx->P * (size_t)G * 4;
    return ok();
  }
  if (which == SKV_WS_APPEND) {
    // Tmax carries the page-id capacity here
    *bytes = 4 * skv::append_ws((long long)B * Hkv, Tmax).words;
    return ok();
  }
  return fail(SKV_ERR_ARG, "skv_workspace_size: unknown kind %d", which);
}

static int fill_alloc_common(skv::AllocParams& p, const skv_ctx* ctx, int B, int Hkv,
                             int64_t Tmax) {
  std::memset(&p, 0, sizeof(p));
  p.B = B;
  p.Hkv = Hkv;
  p.Tmax = Tmax;
  p.P = ctx->P;
  p.outlier = ctx->outlier_protect;
  for (int k = 0; k < 3; ++k) p.kappa[k] = ctx->kappa[k];
  return SKV_OK;
}

int skv_allocate(skv_ctx* ctx, const uint16_t* K, int B, int Hkv, int64_t Tmax,
                 const int32_t* seq_lens, const float* utility, const uint8_t* protect, int mode,
                 const int64_t* budget, const int32_t* quota, const skv_free_lists* free,
                 const skv_pools* pools, uint8_t* tier_out, int32_t* row_of,
                 int32_t* page_indptr, int32_t* page_tier_indptr, uint32_t* page_ids,
                 int64_t page_cap, int32_t* err_word, void* workspace, size_t ws_bytes,
                 void* stream) {
  if (!ctx) return fail(SKV_ERR_ARG, "skv_allocate: null ctx");
  if (B < 0 || Hkv <= 0 || Hkv > 128 || Tmax < 0 || Tmax > (1LL << 23))
    return fail(SKV_ERR_ARG, "skv_allocate: need B >= 0, 0 < Hkv <= 128, 0 <= Tmax <= 2^23");
  if ((long long)B * Hkv > (1 << 30)) return fail(SKV_ERR_ARG, "skv_allocate: too many units");
  if (mode != SKV_MODE_BUDGET && mode != SKV_MODE_QUOTA)
    return fail(SKV_ERR_ARG, "skv_allocate: unknown mode %d", mode);
  if (mode == SKV_MODE_BUDGET && (!utility || !budget || !K))
    return fail(SKV_ERR_ARG, "skv_allocate: budget mode needs K, utility and budget");
  if (mode == SKV_MODE_QUOTA && !quota)
    return fail(SKV_ERR_ARG, "skv_allocate: quota mode needs quota");
  if (!seq_lens || !free || !pools || !tier_out || !row_of || !page_indptr || !err_word)
    return fail(SKV_ERR_ARG, "skv_allocate: null argument");
  if (page_cap > 0 && !page_ids) return fail(SKV_ERR_ARG, "skv_allocate: null page_ids");
  if (!valid_pools(pools, 3))
    return fail(SKV_ERR_ARG, "skv_allocate: pools need 128-byte aligned bases");
  for (int t = 0; t < 3; ++t)
    if (free->len[t] < 0 || (free->len[t] > 0 && !free->ids[t]))
      return fail(SKV_ERR_ARG, "skv_allocate: bad free list %d", t);
  const size_t need = skv::alloc_workspace_bytes(B, Hkv, Tmax);
  if (!workspace || ws_bytes < need)
    return fail(SKV_ERR_ARG, "skv_allocate: workspace of %zu bytes needed", need);
  skv::AllocParams p;
  fill_alloc_common(p, ctx, B, Hkv, Tmax);
  p.K = K;
  p.seq_lens = seq_lens;
  p.utility = utility;
  p.protect = protect;
  p.mode = mode;
  p.budget = budget;
  p.quota = quota;
  for (int t = 0; t < 3; ++t) {
    p.free_ids[t] = free->ids[t];
    p.free_len[t] = free->len[t];
    p.pool[t] = static_cast<uint8_t*>(pools->base[t]);
    p.slots[t] = pools->slots[t];
    p.stride[t] = ctx->stride[t];
    p.payload[t] = (int)ctx->payload[t];
  }
  p.tier_out = tier_out;
  p.row_of = row_of;
  p.indptr = page_indptr;
  p.tier_indptr = page_tier_indptr;
  p.page_ids = page_ids;
  p.page_cap = page_cap;
  p.err = err_word;
  skv::alloc_carve(p, workspace);
  cudaError_t e = skv::launch_allocate(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "skv_allocate launch");
  return ok();
}

int skv_encode(skv_ctx* ctx, const uint16_t* K, const uint16_t* V, int B, int Hkv, int64_t Tmax,
               const int32_t* seq_lens, const uint8_t* tier, const int32_t* row_of,
               const int32_t* page_indptr, const uint32_t* page_ids, const skv_pools* pools,
               int32_t* err_word, void* stream) {
  if (!ctx) return fail(SKV_ERR_ARG, "skv_encode: null ctx");
  if (B < 0 || Hkv <= 0 || Tmax < 0) return fail(SKV_ERR_ARG, "skv_encode: bad sizes");
  if (!K || !V || !seq_lens || !tier || !row_of || !page_indptr || !err_word)
    return fail(SKV_ERR_ARG, "skv_encode: null argument");
  if (!valid_pools(pools, 3)) return fail(SKV_ERR_ARG, "skv_encode: bad pools");
  skv::EncodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.K = K;
  p.V = V;
  p.B = B;
  p.Hkv = Hkv;
  p.Tmax = Tmax;
  p.P = ctx->P;
  p.seq_lens = seq_lens;
  p.tier = tier;
  p.row_of = row_of;
  p.indptr = page_indptr;
  p.ids = page_ids;
  for (int t = 0; t < 3; ++t) {
    p.pool[t] = static_cast<uint8_t*>(pools->base[t]);
    p.slots[t] = pools->slots[t];
    p.stride[t] = ctx->stride[t];
  }
  p.err = err_word;
  p.dense_bf16 = 0;
  p.t0_bf16 = ctx->t0_bf16;
  std::memcpy(p.bx6, ctx->bx6, sizeof(p.bx6));
  std::memcpy(p.by6, ctx->by6, sizeof(p.by6));
  std::memcpy(p.bx4, ctx->bx4, sizeof(p.bx4));
  std::memcpy(p.by4, ctx->by4, sizeof(p.by4));
  std::memcpy(p.bx5, ctx->bx5, sizeof(p.bx5));
  std::memcpy(p.by5, ctx->by5, sizeof(p.by5));
  p.t1_scheme = ctx->t1_scheme;
  p.share_grid = ctx->share_grid;
  cudaError_t e = skv::launch_encode(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "skv_encode launch");
  return ok();
}

int skv_append(skv_ctx* ctx, const uint16_t* K_new, const uint16_t* V_new, int B, int Hkv,
               int64_t Tmax, int32_t* seq_lens, uint8_t* tier, int32_t* row_of,
               int32_t* page_indptr, int32_t* page_tier_indptr, uint32_t* page_ids,
               int64_t page_cap, const skv_pools* pools, const uint32_t* free0,
               int64_t free0_len, int32_t* free0_cursor, int32_t* err_word, void* workspace,
               size_t ws_bytes, void* stream) {
  if (!ctx) return fail(SKV_ERR_ARG, "skv_append: null ctx");
  if (B < 0 || Hkv <= 0 || Tmax <= 0 || page_cap < 0 || free0_len < 0)
    return fail(SKV_ERR_ARG, "skv_append: bad sizes");
  if (!K_new || !V_new || !seq_lens || !tier || !row_of || !page_indptr || !page_tier_indptr ||
      !page_ids || !free0_cursor || !err_word || (free0_len > 0 && !free0))
    return fail(SKV_ERR_ARG, "skv_append: null argument");
  if (!pools || !pools->base[0] || pools->slots[0] < 0) return fail(SKV_ERR_ARG, "skv_append: bad T0 pool");
  if ((long long)B * Hkv > (1LL << 24)) return fail(SKV_ERR_ARG, "skv_append: too many units");
  const size_t need = 4 * skv::append_ws((long long)B * Hkv, page_cap).words;
  if (!workspace || ws_bytes < need)
    return fail(SKV_ERR_ARG, "skv_append: workspace of %zu bytes, %zu needed", ws_bytes, need);
  skv::AppendParams p;
  std::memset(&p, 0, sizeof(p));
  p.K = K_new;
  p.V = V_new;
  p.B = B;
  p.Hkv = Hkv;
  p.Tmax = Tmax;
  p.P = ctx->P;
  p.seq_lens = seq_lens;
  p.tier = tier;
  p.row_of = row_of;
  p.indptr = page_indptr;
  p.tier_indptr = page_tier_indptr;
  p.ids = page_ids;
  p.page_cap = page_cap;
  p.pool0 = static_cast<uint8_t*>(pools->base[0]);
  p.slots0 = pools->slots[0];
  p.stride0 = ctx->stride[0];
  p.free0 = free0;
  p.free0_len = free0_len;
  p.free0_cursor = free0_cursor;
  p.err = err_word;
  p.ws = static_cast<int32_t*>(workspace);
  p.t0_bf16 = ctx->t0_bf16;
  cudaError_t e = skv::launch_append(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "skv_append launch");
  return ok();
}

int skv_retier_workspace_size(const skv_ctx* ctx, int B, int Hkv, int64_t Tmax,
                              int64_t page_cap, size_t* bytes) {
  if (!ctx || !bytes) return fail(SKV_ERR_ARG, "skv_retier_workspace_size: null argument");
  if (B < 0 || Hkv <= 0 || Tmax < 0 || page_cap < 0)
    return fail(SKV_ERR_ARG, "skv_retier_workspace_size: bad sizes");
  *bytes = skv::retier_workspace_bytes(B, Hkv, Tmax, page_cap);
  return ok();
}

int skv_retier(skv_ctx* ctx, int B, int Hkv, int64_t Tmax, const int32_t* seq_lens,
               const float* utility, const uint8_t* demote, const int64_t* budget,
               const skv_free_lists* free, int32_t* free_cursor, const skv_pools* pools,
               uint8_t* tier, int32_t* row_of, int32_t* page_indptr,
               int32_t* page_tier_indptr, uint32_t* page_ids, int64_t page_cap,
               uint32_t* released, int32_t* n_released, int32_t* err_word, void* workspace,
               size_t ws_bytes, void* stream) {
  if (!ctx) return fail(SKV_ERR_ARG, "skv_retier: null ctx");
  if (ctx->t0_bf16)
    return fail(SKV_ERR_ARG, "skv_retier: the demoted rows' exact fp16 keys are not in bf16 T0 pages");
  if (B < 0 || Hkv <= 0 || Hkv > 128 || Tmax < 0 || Tmax > (1LL << 23) || page_cap < 0 ||
      page_cap > 0x7FFFFFFFLL)
    return fail(SKV_ERR_ARG, "skv_retier: need B >= 0, 0 < Hkv <= 128, 0 <= Tmax <= 2^23");
  if ((long long)B * Hkv > (1 << 24)) return fail(SKV_ERR_ARG, "skv_retier: too many units");
  if ((long long)B * Hkv * Tmax > 0xFFFFFFFFLL)  // rows to rewrite are listed by 32-bit index
    return fail(SKV_ERR_ARG, "skv_retier: B * Hkv * Tmax must be below 2^32");
  if (!seq_lens || !utility || !demote || !budget || !free || !free_cursor || !tier ||
      !row_of || !page_indptr || !page_tier_indptr || !released || !n_released || !err_word)
    return fail(SKV_ERR_ARG, "skv_retier: null argument");
  if (page_cap > 0 && !page_ids) return fail(SKV_ERR_ARG, "skv_retier: null page_ids");
  if (!valid_pools(pools, 3))
    return fail(SKV_ERR_ARG, "skv_retier: pools need 128-byte aligned bases");
  for (int t = 0; t < 3; ++t)
    if (free->len[t] < 0 || (free->len[t] > 0 && !free->ids[t]))
      return fail(SKV_ERR_ARG, "skv_retier: bad free list %d", t);
  const size_t need = skv::retier_workspace_bytes(B, Hkv, Tmax, page_cap);
  if (!workspace || ws_bytes < need)
    return fail(SKV_ERR_ARG, "skv_retier: workspace of %zu bytes needed", need);
  skv::AllocParams p;
  fill_alloc_common(p, ctx, B, Hkv, Tmax);
  p.seq_lens = seq_lens;
  p.utility = utility;
  p.demote = demote;
  p.mode = SKV_MODE_BUDGET;
  p.budget = budget;
  for (int t = 0; t < 3; ++t) {
    p.free_ids[t] = free->ids[t];
    p.free_len[t] = free->len[t];
    p.pool[t] = static_cast<uint8_t*>(pools->base[t]);
    p.slots[t] = pools->slots[t];
    p.stride[t] = ctx->stride[t];
    p.payload[t] = (int)ctx->payload[t];
  }
  p.tier_out = tier;
  p.row_of = row_of;
  p.indptr = page_indptr;
  p.tier_indptr = page_tier_indptr;
  p.page_ids = page_ids;
  p.page_cap = page_cap;
  p.cursor = free_cursor;
  p.released = released;
  p.n_released = n_released;
  p.err = err_word;
  skv::retier_carve(p, workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = skv::launch_retier_plan(p, st);
  if (e != cudaSuccess) return cuda_fail(e, "skv_retier plan");
  skv::TranscodeParams tp;
  std::memset(&tp, 0, sizeof(tp));
  tp.B = B;
  tp.Hkv = Hkv;
  tp.Tmax = Tmax;
  tp.P = ctx->P;
  tp.seq_lens = seq_lens;
  tp.tier = tier;
  tp.row_of = row_of;
  tp.indptr = page_indptr;
  tp.tier_indptr = page_tier_indptr;
  tp.ids = page_ids;
  tp.keep = p.keep;
  tp.page_cap = page_cap;
  tp.tier_old = p.tier_old;
  tp.row_old = p.row_old;
  tp.indptr_old = p.indptr_old;
  tp.ids_old = p.ids_old;
  for (int t = 0; t < 3; ++t) {
    tp.pool[t] = p.pool[t];
    tp.slots[t] = p.slots[t];
    tp.stride[t] = p.stride[t];
  }
  tp.err = err_word;
  // the key array and the histogram are free once the tiers are decided
  tp.list = reinterpret_cast<uint32_t*>(p.keyw);
  tp.count = p.hist;
  std::memcpy(tp.bx6, ctx->bx6, sizeof(tp.bx6));
  std::memcpy(tp.by6, ctx->by6, sizeof(tp.by6));
  std::memcpy(tp.bx4, ctx->bx4, sizeof(tp.bx4));
  std::memcpy(tp.by4, ctx->by4, sizeof(tp.by4));
  std::memcpy(tp.bx5, ctx->bx5, sizeof(tp.bx5));
  std::memcpy(tp.by5, ctx->by5, sizeof(tp.by5));
  tp.t1_scheme = ctx->t1_scheme;
  tp.share_grid = ctx->share_grid;
  e = skv::launch_transcode(tp, st);
  if (e != cudaSuccess) return cuda_fail(e, "skv_retier transcode");
  return ok();
}

static int decode_common(skv_ctx* ctx, const void* q, int q_dtype, int B, int Hq, int Hkv,
                         const int32_t* page_indptr, const int32_t* page_tier_indptr,
                         const uint32_t* page_ids, const void* pool[3],
                         const long long slots[3], bool dense, float* out, float* lse,
                         int32_t* err_word, void* workspace, size_t ws_bytes, int num_splits,
                         void* stream, const char* name, float* logits = nullptr,
                         long long logit_rows = 0) {
  if (!ctx) return fail(SKV_ERR_ARG, "%s: null ctx", name);
  if (B < 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0)
    return fail(SKV_ERR_ARG, "%s: need B >= 0 and Hq a multiple of Hkv", name);
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4) return fail(SKV_ERR_ARG, "%s: Hq/Hkv must be 1, 2 or 4", name);
  if (q_dtype != SKV_Q_BF16 && q_dtype != SKV_Q_FP16)
    return fail(SKV_ERR_ARG, "%s: unknown q dtype %d", name, q_dtype);
  if (num_splits < 0) return fail(SKV_ERR_ARG, "%s: num_splits < 0", name);
  if (B == 0) return ok();
  if (!q || !page_indptr || !out || !err_word)
    return fail(SKV_ERR_ARG, "%s: null argument", name);
  size_t need = 0;
  skv_workspace_size(ctx, dense ? SKV_WS_DENSE_DECODE : SKV_WS_DECODE, B, Hkv, Hq, 0, num_splits,
                     &need);
  if (!workspace || ws_bytes < need)
    return fail(SKV_ERR_ARG, "%s: workspace of %zu bytes needed", name, need);
  skv::DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q;
  p.q_bf16 = q_dtype == SKV_Q_BF16;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.indptr = page_indptr;
  p.tier_indptr = page_tier_indptr;
  p.ids = page_ids;
  for (int t = 0; t < 3; ++t) {
    p.pool[t] = static_cast<const uint8_t*>(pool[t]);
    p.slots[t] = slots[t];
    const int ti = dense ? 3 : t;
    p.stride[t] = ctx->stride[ti];
    p.payload[t] = (int)ctx->payload[ti];
    p.cost[t] = (int)split_cost(ctx, ti);
  }
  p.out = out;
  p.lse = lse;
  p.err = err_word;
  p.part = static_cast<float*>(workspace);
  p.logits = logits;
  p.logit_rows = logit_rows;
  p.S = decode_splits(ctx, num_splits);
  p.P = ctx->P;
  p.log2P = ctx->log2P;
  long long max_pay = p.payload[0];
  if (!dense) max_pay = std::max(max_pay, (long long)std::max(p.payload[1], p.payload[2]));
  const long long max_item = (skv::kDecodeItemRows / p.P) * max_pay;
  if (!skv::decode_smem_ok(G, dense, (int)ctx->smem_optin, (int)max_item))
    return fail(SKV_ERR_ARG, "%s: not enough shared memory per block", name);
  p.smem_bytes = (int)ctx->smem_optin;
  p.qk_scale_log2 = (float)(1.4426950408889634 / std::sqrt(128.0));
  std::memcpy(p.cos6, ctx->cos6, sizeof(p.cos6));
  std::memcpy(p.sin6, ctx->sin6, sizeof(p.sin6));
  std::memcpy(p.cos4, ctx->cos4, sizeof(p.cos4));
  std::memcpy(p.sin4, ctx->sin4, sizeof(p.sin4));
  std::memcpy(p.cos5, ctx->cos5, sizeof(p.cos5));
  std::memcpy(p.sin5, ctx->sin5, sizeof(p.sin5));
  p.t1_scheme = ctx->t1_scheme;
  p.share_grid = ctx->share_grid;
  p.t0_bf16 = dense ? 0 : ctx->t0_bf16;
  p.dynamic = ctx->deterministic ? 0 : 1;
  p.wait_limit = ctx->wait_limit > 0 ? ctx->wait_limit : 2000000000LL;
  cudaError_t e =
      skv::launch_decode(p, G, dense, static_cast<cudaStream_t>(stream), ctx->profile_event);
  if (e != cudaSuccess) return cuda_fail(e, name);
  return ok();
}

int skv_decode_attention(skv_ctx* ctx, const void* q, int q_dtype, int B, int Hq, int Hkv,
                         const int32_t* page_indptr, const int32_t* page_tier_indptr,
                         const uint32_t* page_ids, const skv_pools* pools, float* out,
                         float* lse, int32_t* err_word, void* workspace, size_t ws_bytes,
                         int num_splits, void* stream) {
  if (!valid_pools(pools, 3)) return fail(SKV_ERR_ARG, "skv_decode_attention: bad pools");
  const void* pool[3] = {pools->base[0], pools->base[1], pools->base[2]};
  const long long slots[3] = {pools->slots[0], pools->slots[1], pools->slots[2]};
  return decode_common(ctx, q, q_dtype, B, Hq, Hkv, page_indptr, page_tier_indptr, page_ids, pool,
                       slots, false, out,
                       lse, err_word, workspace, ws_bytes, num_splits, stream,
                       "skv_decode_attention");
}

// The stream operations of one host step: q copy, decode (+ merge), the
// result copies (one when packed), the error word's copy and its reset.
static int host_step_ops(skv_ctx* ctx, const void* q_host, int q_dtype, int B, int Hq, int Hkv,
                         const int32_t* page_indptr, const int32_t* page_tier_indptr,
                         const uint32_t* page_ids, const skv_pools* pools, void* q_dev,
                         float* out_dev, float* lse_dev, float* out_host, float* lse_host,
                         bool packed, int32_t* err_word, int32_t* err_dst, void* workspace,
                         size_t ws_bytes, int num_splits, void* stream, const char* name) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t qn = (size_t)B * Hq * 128 * 2, on = (size_t)B * Hq * 128 * 4, ln = (size_t)B * Hq * 4;
  // a copy, not reads of mapped host memory by the decode: those made the
  // step 8.5 us slower (99 against 90.5 us on the 128K store)
  cudaError_t e = cudaMemcpyAsync(q_dev, q_host, qn, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "skv_decode_attention_host: copy of q");
  const void* pool[3] = {pools->base[0], pools->base[1], pools->base[2]};
  const long long slots[3] = {pools->slots[0], pools->slots[1], pools->slots[2]};
  int rc = decode_common(ctx, q_dev, q_dtype, B, Hq, Hkv, page_indptr, page_tier_indptr, page_ids,
                         pool, slots, false, out_dev, lse_dev, err_word, workspace, ws_bytes,
                         num_splits, stream, name);
  if (rc != SKV_OK) return rc;
  // copies, not kernel stores into mapped host memory: writing the results
  // through the mapping made the step slower (103 against 98 us on the 128K store)
  if (packed) {
    e = cudaMemcpyAsync(out_host, out_dev, on + ln, cudaMemcpyDeviceToHost, s);
  } else {
    e = cudaMemcpyAsync(out_host, out_dev, on, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(lse_host, lse_dev, ln, cudaMemcpyDeviceToHost, s);
  }
  // the error word rides along with the results, and is reset on the stream
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(err_dst, err_word, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(err_word, 0, sizeof(int32_t), s);
  if (e != cudaSuccess) return cuda_fail(e, "skv_decode_attention_host: copy of the results");
  return SKV_OK;
}

int skv_decode_attention_host(skv_ctx* ctx, const void* q_host, int q_dtype, int B, int Hq,
                              int Hkv, const int32_t* page_indptr,
                              const int32_t* page_tier_indptr, const uint32_t* page_ids,
                              const skv_pools* pools, void* q_dev, float* out_dev, float* lse_dev,
                              float* out_host, float* lse_host, int32_t* err_word,
                              void* workspace, size_t ws_bytes, int num_splits, void* stream) {
  static const char* name = "skv_decode_attention_host";
  if (!ctx) return fail(SKV_ERR_ARG, "%s: null ctx", name);
  if (B < 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0)
    return fail(SKV_ERR_ARG, "%s: need B >= 0 and Hq a multiple of Hkv", name);
  if (B == 0) return ok();
  const bool packed = lse_dev == nullptr && lse_host == nullptr;  // lse follows out
  if (!q_host || !q_dev || !out_dev || !out_host || !err_word ||
      (!packed && (!lse_dev || !lse_host)))
    return fail(SKV_ERR_ARG, "%s: null argument", name);
  if (!valid_pools(pools, 3)) return fail(SKV_ERR_ARG, "%s: bad pools", name);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);  // the first call allocates the word
    if (!ctx->err_host) {
      e = cudaMallocHost(&ctx->err_host, sizeof(int32_t));
      if (e != cudaSuccess) return cuda_fail(e, "skv_decode_attention_host: pinned error word");
      *ctx->err_host = 0;
    }
  }
  const size_t on_f = (size_t)B * Hq * 128;
  if (packed) {
    lse_dev = out_dev + on_f;
    lse_host = out_host + on_f;
  }
  // one eager step: a CUDA graph of the same operations, captured once and
  // replayed, measured 5 us slower a step (91.7 against 86.7 us)
  const int rc = host_step_ops(ctx, q_host, q_dtype, B, Hq, Hkv, page_indptr, page_tier_indptr,
                               page_ids, pools, q_dev, out_dev, lse_dev, out_host, lse_host,
                               packed, err_word, ctx->err_host, workspace, ws_bytes, num_splits,
                               stream, name);
  if (rc != SKV_OK) return rc;
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "skv_decode_attention_host: stream synchronize");
  const int32_t v = *ctx->err_host;
  if (v != 0) return fail(v, "%s: device reported error %d", name, v);
  return ok();
}

int skv_decode_attention_host_pipelined(skv_ctx* ctx, const void* q_host, int q_dtype, int B,
                                        int Hq, int Hkv, const int32_t* page_indptr,
                                        const int32_t* page_tier_indptr,
                                        const uint32_t* page_ids, const skv_pools* pools,
                                        void* q_dev, float* res_dev, float* res_host,
                                        void* workspace, size_t ws_bytes, int num_splits,
                                        void* stream) {
  static const char* name = "skv_decode_attention_host_pipelined";
  if (!ctx) return fail(SKV_ERR_ARG, "%s: null ctx", name);
  if (B <= 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0)
    return fail(SKV_ERR_ARG, "%s: need B > 0 and Hq a multiple of Hkv", name);
  if (!q_host || !q_dev || !res_dev || !res_host)
    return fail(SKV_ERR_ARG, "%s: null argument", name);
  if (!valid_pools(pools, 3)) return fail(SKV_ERR_ARG, "%s: bad pools", name);
  if (ctx->pipe_pending && ctx->pipe_stream != stream)
    return fail(SKV_ERR_ARG, "%s: a step is pending on another stream (drain it first)", name);
  cudaError_t e = cudaSuccess;
  if (!ctx->pipe_err) {  // first use: the slots' words, events and copy streams
    if ((e = cudaMallocHost(&ctx->pipe_err, 2 * sizeof(int32_t))) != cudaSuccess ||
        (e = cudaMalloc(&ctx->pipe_err_dev, 2 * sizeof(int32_t))) != cudaSuccess ||
        (e = cudaMemset(ctx->pipe_err_dev, 0, 2 * sizeof(int32_t))) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&ctx->pipe_in, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&ctx->pipe_out, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e, "skv_decode_attention_host_pipelined: set-up");
    ctx->pipe_err[0] = ctx->pipe_err[1] = 0;
    for (int i = 0; i < 2; ++i)
      if ((e = cudaEventCreateWithFlags(&ctx->pipe_ev_q[i], cudaEventDisableTiming)) !=
              cudaSuccess ||
          (e = cudaEventCreateWithFlags(&ctx->pipe_ev_d[i], cudaEventDisableTiming)) !=
              cudaSuccess ||
          (e = cudaEventCreateWithFlags(&ctx->pipe_ev_r[i], cudaEventDisableTiming)) != cudaSuccess)
        return cuda_fail(e, "skv_decode_attention_host_pipelined: events");
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int slot = (int)(ctx->pipe_n & 1);
  const size_t qn = (size_t)B * Hq * 128 * 2, rn = (size_t)B * Hq * 129;
  uint8_t* qd = static_cast<uint8_t*>(q_dev) + slot * qn;
  float* rd = res_dev + slot * rn;
  int32_t* ed = ctx->pipe_err_dev + slot;
  // q in on the copy-in stream (it may run while the previous decode does)
  if ((e = cudaMemcpyAsync(qd, q_host, qn, cudaMemcpyHostToDevice, ctx->pipe_in)) != cudaSuccess ||
      (e = cudaEventRecord(ctx->pipe_ev_q[slot], ctx->pipe_in)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(s, ctx->pipe_ev_q[slot], 0)) != cudaSuccess)
    return cuda_fail(e, "skv_decode_attention_host_pipelined: q copy");
  const void* pool[3] = {pools->base[0], pools->base[1], pools->base[2]};
  const long long slots[3] = {pools->slots[0], pools->slots[1], pools->slots[2]};
  int rc = decode_common(ctx, qd, q_dtype, B, Hq, Hkv, page_indptr, page_tier_indptr, page_ids,
                         pool, slots, false, rd, rd + (size_t)B * Hq * 128, ed, workspace,
                         ws_bytes, num_splits, stream, name);
  if (rc != SKV_OK) return rc;
  // out + lse and the error word out on the copy-out stream, behind the decode
  if ((e = cudaEventRecord(ctx->pipe_ev_d[slot], s)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(ctx->pipe_out, ctx->pipe_ev_d[slot], 0)) != cudaSuccess ||
      (e = cudaMemcpyAsync(res_host, rd, rn * sizeof(float), cudaMemcpyDeviceToHost,
                           ctx->pipe_out)) != cudaSuccess ||
      (e = cudaMemcpyAsync(&ctx->pipe_err[slot], ed, sizeof(int32_t), cudaMemcpyDeviceToHost,
                           ctx->pipe_out)) != cudaSuccess ||
      (e = cudaMemsetAsync(ed, 0, sizeof(int32_t), ctx->pipe_out)) != cudaSuccess ||
      (e = cudaEventRecord(ctx->pipe_ev_r[slot], ctx->pipe_out)) != cudaSuccess)
    return cuda_fail(e, "skv_decode_attention_host_pipelined: result copies");
  const bool had_prev = ctx->pipe_pending;
  ctx->pipe_n += 1;
  ctx->pipe_pending = true;
  ctx->pipe_stream = stream;
  if (!had_prev) return ok();
  // the previous step: its results are in the host buffer of the previous call
  e = cudaEventSynchronize(ctx->pipe_ev_r[slot ^ 1]);
  if (e != cudaSuccess) return cuda_fail(e, "skv_decode_attention_host_pipelined: event wait");
  const int32_t v = ctx->pipe_err[slot ^ 1];
  if (v != 0) return fail(v, "%s: the previous step reported error %d", name, v);
  return ok();
}

int skv_decode_attention_host_drain(skv_ctx* ctx) {
  if (!ctx) return fail(SKV_ERR_ARG, "skv_decode_attention_host_drain: null ctx");
  if (!ctx->pipe_pending) return ok();
  const int slot = (int)((ctx->pipe_n - 1) & 1);
  ctx->pipe_pending = false;
  cudaError_t e = cudaEventSynchronize(ctx->pipe_ev_r[slot]);
  if (e != cudaSuccess) return cuda_fail(e, "skv_decode_attention_host_drain: event wait");
  const int32_t v = ctx->pipe_err[slot];
  if (v != 0) return fail(v, "skv_decode_attention_host_drain: the last step reported error %d", v);
  return ok();
}

int skv_merge_partials(skv_ctx* ctx, int R, int64_t n, const float* out_parts,
                       const float* lse_parts, int64_t rank_stride, float* out, float* lse,
                       void* stream) {
  static const char* name = "skv_merge_partials";
  if (!ctx) return fail(SKV_ERR_ARG, "%s: null ctx", name);
  if (R <= 0 || n < 0 || n > 0x7FFFFFFFLL)
    return fail(SKV_ERR_ARG, "%s: need R > 0 and 0 <= n < 2^31", name);
  if (n == 0) return ok();
  if (!out_parts || !lse_parts || !out) return fail(SKV_ERR_ARG, "%s: null argument", name);
  if (R > 1 && rank_stride < n) return fail(SKV_ERR_ARG, "%s: rank_stride < n", name);
  if ((reinterpret_cast<uintptr_t>(out_parts) & 7) || (reinterpret_cast<uintptr_t>(out) & 7) ||
      (rank_stride & 1))
    return fail(SKV_ERR_ARG, "%s: out_parts, out and rank_stride must be 8-byte aligned", name);
  cudaError_t e = skv::launch_merge_partials(R, n, out_parts, lse_parts, rank_stride, out, lse,
                                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, name);
  return ok();
}

int skv_decode_utility(skv_ctx* ctx, const void* q, int q_dtype, int B, int Hq, int Hkv,
                       const int32_t* page_indptr, const int32_t* page_tier_indptr,
                       const uint32_t* page_ids, int64_t page_cap, const skv_pools* pools,
                       int64_t Tmax, const int32_t* seq_lens, const uint8_t* tier,
                       const int32_t* row_of, float gamma, float* utility, float* out, float* lse,
                       int32_t* err_word, void* workspace, size_t ws_bytes, int num_splits,
                       void* stream) {
  static const char* name = "skv_decode_utility";
  if (!ctx) return fail(SKV_ERR_ARG, "%s: null ctx", name);
  if (B < 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0 || Tmax < 0 || page_cap < 0 ||
      num_splits < 0)
    return fail(SKV_ERR_ARG, "%s: bad sizes", name);
  if (B == 0) return ok();
  if (!seq_lens || !tier || !row_of || !utility || !lse)
    return fail(SKV_ERR_ARG, "%s: null argument", name);
  if (!valid_pools(pools, 3)) return fail(SKV_ERR_ARG, "%s: bad pools", name);
  size_t need = 0;
  int rc = skv_workspace_size(ctx, SKV_WS_DECODE_UTILITY, B, Hkv, Hq, page_cap, num_splits, &need);
  if (rc != SKV_OK) return rc;
  if (!workspace || ws_bytes < need)
    return fail(SKV_ERR_ARG, "%s: workspace of %zu bytes needed", name, need);
  const int G = Hq / Hkv;
  const size_t at = decode_utility_logits_at(decode_splits(ctx, num_splits), (long long)B * Hkv, G);
  float* logits = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + at);
  const long long rows = (long long)page_cap * ctx->P;
  const void* pool[3] = {pools->base[0], pools->base[1], pools->base[2]};
  const long long slots[3] = {pools->slots[0], pools->slots[1], pools->slots[2]};
  rc = decode_common(ctx, q, q_dtype, B, Hq, Hkv, page_indptr, page_tier_indptr, page_ids, pool,
                     slots, false, out, lse, err_word, workspace, at, num_splits, stream, name,
                     logits, rows);
  if (rc != SKV_OK) return rc;
  skv::UtilityParams u;
  u.logits = logits;
  u.logit_rows = rows;
  u.lse = lse;
  u.seq_lens = seq_lens;
  u.tier = tier;
  u.row_of = row_of;
  u.indptr = page_indptr;
  u.B = B;
  u.Hkv = Hkv;
  u.G = G;
  u.P = ctx->P;
  u.Tmax = Tmax;
  u.gamma = gamma;
  u.utility = utility;
  u.err = err_word;
  cudaError_t e = skv::launch_utility(u, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "skv_decode_utility: utility update");
  return ok();
}

int skv_dense_decode_bf16(skv_ctx* ctx, const void* q, int q_dtype, int B, int Hq, int Hkv,
                          const int32_t* page_indptr, const uint32_t* page_ids, const void* pool,
                          int64_t pool_slots, float* out, float* lse, int32_t* err_word,
                          void* workspace, size_t ws_bytes, int num_splits, void* stream) {
  if ((reinterpret_cast<uintptr_t>(pool) & 127) != 0 || pool_slots < 0)
    return fail(SKV_ERR_ARG, "skv_dense_decode_bf16: bad pool");
  const void* pools[3] = {pool, nullptr, nullptr};
  const long long slots[3] = {pool_slots, 0, 0};
  return decode_common(ctx, q, q_dtype, B, Hq, Hkv, page_indptr, nullptr, page_ids, pools, slots,
                       true, out,
                       lse, err_word, workspace, ws_bytes, num_splits, stream,
                       "skv_dense_decode_bf16");
}

int skv_dense_pack_bf16(skv_ctx* ctx, const uint16_t* K, const uint16_t* V, int B, int Hkv,
                        int64_t Tmax, const int32_t* seq_lens, const uint32_t* free_ids,
                        int64_t free_len, void* pool, int64_t pool_slots, int32_t* page_indptr,
                        uint32_t* page_ids, int64_t page_cap, int32_t* err_word, void* workspace,
                        size_t ws_bytes, void* stream) {
  if (!ctx) return fail(SKV_ERR_ARG, "skv_dense_pack_bf16: null ctx");
  if (B < 0 || Hkv <= 0 || Hkv > 128 || Tmax < 0)
    return fail(SKV_ERR_ARG, "skv_dense_pack_bf16: bad sizes");
  if (!K || !V || !seq_lens || !page_indptr || !err_word || (free_len > 0 && !free_ids))
    return fail(SKV_ERR_ARG, "skv_dense_pack_bf16: null argument");
  if ((reinterpret_cast<uintptr_t>(pool) & 127) != 0 || pool_slots < 0)
    return fail(SKV_ERR_ARG, "skv_dense_pack_bf16: bad pool");
  const size_t need = skv::alloc_workspace_bytes(B, Hkv, Tmax);
  if (!workspace || ws_bytes < need)
    return fail(SKV_ERR_ARG, "skv_dense_pack_bf16: workspace of %zu bytes needed", need);
  skv::AllocParams a;
  fill_alloc_common(a, ctx, B, Hkv, Tmax);
  a.seq_lens = seq_lens;
  a.free_ids[0] = free_ids;
  a.free_len[0] = free_len;
  a.pool[0] = static_cast<uint8_t*>(pool);
  a.slots[0] = pool_slots;
  a.stride[0] = ctx->stride[3];
  a.payload[0] = (int)ctx->payload[3];
  a.indptr = page_indptr;
  a.page_ids = page_ids;
  a.page_cap = page_cap;
  a.err = err_word;
  skv::alloc_carve(a, workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = skv::launch_dense_plan(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "skv_dense_pack_bf16 plan");
  skv::EncodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.K = K;
  p.V = V;
  p.B = B;
  p.Hkv = Hkv;
  p.Tmax = Tmax;
  p.P = ctx->P;
  p.seq_lens = seq_lens;
  p.indptr = page_indptr;
  p.ids = page_ids;
  p.pool[0] = static_cast<uint8_t*>(pool);
  p.slots[0] = pool_slots;
  p.stride[0] = ctx->stride[3];
  p.err = err_word;
  p.dense_bf16 = 1;
  e = skv::launch_encode(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "skv_dense_pack_bf16 encode");
  return ok();
}

int skv_decode_attention_static(skv_ctx* ctx, const void* q, int q_dtype, int B, int Hq,
                                int Hkv, const int32_t* page_indptr,
                                const int32_t* page_tier_indptr, const uint32_t* page_ids,
                                const skv_pools* pools, float* out, float* lse,
                                int32_t* err_word, int num_splits, void* stream) {
  static const char* name = "skv_decode_attention_static";
  if (!ctx) return fail(SKV_ERR_ARG, "%s: null ctx", name);
  if (B < 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0 || num_splits < 0)
    return fail(SKV_ERR_ARG, "%s: need B >= 0, Hq a multiple of Hkv, num_splits >= 0", name);
  if (B == 0) return ok();
  size_t need = 0;
  const int rc = skv_workspace_size(ctx, SKV_WS_DECODE, B, Hkv, Hq, 0, num_splits, &need);
  if (rc != SKV_OK) return rc;
  if (need > kStaticScratchBytes)
    return fail(SKV_ERR_ARG,
                "%s: this call needs %zu bytes of scratch; the static scratch holds %zu "
                "(use skv_decode_attention with a workspace)",
                name, need, kStaticScratchBytes);
  if (!valid_pools(pools, 3)) return fail(SKV_ERR_ARG, "%s: bad pools", name);
  void* scratch = nullptr;
  cudaError_t e = static_scratch(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "skv_decode_attention_static: scratch address");
  const void* pool[3] = {pools->base[0], pools->base[1], pools->base[2]};
  const long long slots[3] = {pools->slots[0], pools->slots[1], pools->slots[2]};
  return decode_common(ctx, q, q_dtype, B, Hq, Hkv, page_indptr, page_tier_indptr, page_ids, pool,
                       slots, false, out, lse, err_word, scratch, kStaticScratchBytes, num_splits,
                       stream, name);
}

int skv_set_profile_event(skv_ctx* ctx, void* event) {
  if (!ctx) return fail(SKV_ERR_ARG, "skv_set_profile_event: null ctx");
  ctx->profile_event = static_cast<cudaEvent_t>(event);
  return ok();
}

int skv_set_wait_limit(skv_ctx* ctx, int64_t cycles) {
  if (!ctx || cycles < 0) return fail(SKV_ERR_ARG, "skv_set_wait_limit: null ctx or negative limit");
  ctx->wait_limit = cycles;
  return ok();
}

int skv_check(skv_ctx* ctx, int32_t* err_word, void* stream) {
  if (!ctx || !err_word) return fail(SKV_ERR_ARG, "skv_check: null argument");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "skv_check: stream synchronize");
  int32_t v = 0;
  e = cudaMemcpy(&v, err_word, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "skv_check: read error word");
  e = cudaMemset(err_word, 0, sizeof(int32_t));
  if (e != cudaSuccess) return cuda_fail(e, "skv_check: reset error word");
  if (v != 0) {
    static const char* names[] = {"ok", "argument", "budget", "pool", "corrupt page table",
                                  "cuda", "timeout"};
    return fail(v, "device reported error %d (%s)", v, (v >= 0 && v <= 6) ? names[v] : "?");
  }
  return ok();
}

}  // extern "C"
