// C-ABI entry points of libps: argument validation, status codes, tensor-map encoding and
// kernel launches.  The declarations and their contracts are in include/ps.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>

#include <mutex>
#include <string>

#include "../../include/ps.h"
#include "ps_internal.h"
#include "ps_ranges.cuh"

namespace ps {
// ps_diag.cu: one CTA whose bounded wait runs out (ps_check_wait_timeout).
cudaError_t launch_wait_timeout(int32_t* status, cudaStream_t stream);
}  // namespace ps

namespace ps {

namespace {
thread_local std::string g_last_error;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Validates the geometry shared by every call.
int check_params(const ps_params* prm, bool need_window) {
  if (!prm) return fail(PS_ERR_INVALID_ARG, "params is NULL");
  if (prm->reserved != 0 || prm->reserved2 != 0)
    return fail(PS_ERR_INVALID_ARG, "params reserved fields must be 0");
  if (prm->head_dim != kHeadDim)
    return fail(PS_ERR_UNSUPPORTED, "head_dim must be 128 (the only head size this library implements)");
  if (prm->n_q_heads < 1 || prm->n_kv_heads < 1)
    return fail(PS_ERR_INVALID_ARG, "n_q_heads and n_kv_heads must be >= 1");
  if (prm->n_q_heads % prm->n_kv_heads != 0)
    return fail(PS_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads");
  if (need_window) {
    if (prm->l_prefix < 0) return fail(PS_ERR_INVALID_ARG, "l_prefix must be >= 0");
    if (prm->window < 1) return fail(PS_ERR_INVALID_ARG, "window must be >= 1");
  }
  if (!(prm->rope_theta > 0.0) || !isfinite(prm->rope_theta))
    return fail(PS_ERR_INVALID_ARG, "rope_theta must be finite and > 0");
  if (!(prm->softmax_scale >= 0.f) || !isfinite(prm->softmax_scale))
    return fail(PS_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  return PS_OK;
}

float resolve_scale(const ps_params* prm) {
  return prm->softmax_scale > 0.f ? prm->softmax_scale
                                  : static_cast<float>(1.0 / sqrt(double(prm->head_dim)));
}

int check_ptr(const void* p, const char* name, bool nullable = false) {
  if (!p) {
    if (nullable) return PS_OK;
    return fail(PS_ERR_INVALID_ARG, std::string(name) + " is NULL");
  }
  if (!aligned16(p)) return fail(PS_ERR_INVALID_ARG, std::string(name) + " is not 16-byte aligned");
  return PS_OK;
}

#define PS_TRY(expr)             \
  do {                           \
    const int rc_ = (expr);      \
    if (rc_ != PS_OK) return rc_; \
  } while (0)

}  // namespace

int fail(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

int check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return PS_OK;
  return fail(PS_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

bool make_map_3d(CUtensorMap* map, const void* base, uint64_t x, uint64_t y, uint64_t z,
                 uint32_t box_x, uint32_t box_y) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    fail(PS_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (no CUDA driver?)");
    return false;
  }
  const cuuint64_t dims[3] = {x, y, z};
  const cuuint64_t strides[2] = {x * 2, x * y * 2};
  const cuuint32_t box[3] = {box_x, box_y, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[160];
    snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled failed (%d) dims %llu x %llu x %llu",
             int(r), (unsigned long long)x, (unsigned long long)y, (unsigned long long)z);
    fail(PS_ERR_CUDA, buf);
    return false;
  }
  return true;
}

bool make_map_4d(CUtensorMap* map, const void* base, const uint64_t dims[4],
                 const uint32_t box[4]) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    fail(PS_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (no CUDA driver?)");
    return false;
  }
  const cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
  const cuuint64_t strides[3] = {dims[0] * 2, dims[0] * dims[1] * 2,
                                 dims[0] * dims[1] * dims[2] * 2};
  const cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), d,
                        strides, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fail(PS_ERR_CUDA, "cuTensorMapEncodeTiled (4-D) failed (" + std::to_string(int(r)) + ")");
    return false;
  }
  return true;
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace ps

namespace ps {
namespace {
// Shared-prefix decode workspace: [window-pass split-K partials][prefix partials o]
// [prefix partials lse2], each part 256-byte aligned.
struct SharedPrefixLayout {
  size_t dec, o, lse, total;
  int splits;
};
SharedPrefixLayout shared_prefix_layout(const ps_params* p, int64_t batch, int64_t gsize) {
  SharedPrefixLayout L;
  L.splits = shared_prefix_splits(batch, gsize, p->n_q_heads, p->n_kv_heads, p->l_prefix);
  L.dec = (decode_workspace_bytes(batch, p->n_kv_heads, (int64_t)p->l_prefix + p->window, true) +
           255) & ~size_t(255);
  L.o = (size_t(L.splits) * batch * p->n_q_heads * kHeadDim * 4 + 255) & ~size_t(255);
  L.lse = (size_t(L.splits) * batch * p->n_q_heads * 4 + 255) & ~size_t(255);
  L.total = L.dec + L.o + L.lse;
  return L;
}
// Process-unique id of the current context (cuCtxGetId), 0 if the CUDA driver cannot tell.
// The primary context keeps its handle across cudaDeviceReset, but not its id.
unsigned long long current_context_id() {
  using CtxGetCurrentFn = CUresult (*)(CUcontext*);
  using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx)
    get_id(ctx, &id);
  return id;
}

// Side stream (one per device and context, created on first use) on which the shared-prefix
// pass runs concurrently with the window decode.  A stream of a context that has since been
// destroyed (cudaDeviceReset) is abandoned, not reused: its handle is no longer valid.
cudaStream_t side_stream(int* rc) {
  static std::mutex mu;
  static cudaStream_t streams[64] = {nullptr};
  static unsigned long long owner[64] = {0};
  int dev = 0;
  *rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
  if (*rc != PS_OK) return nullptr;
  if (dev < 0 || dev >= 64) {
    *rc = fail(PS_ERR_UNSUPPORTED, "device index above 63");
    return nullptr;
  }
  // the current context: the caller's device buffers live in it
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev] || owner[dev] != ctx) {
    *rc = check_cuda(cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking),
                     "cudaStreamCreateWithFlags");
    if (*rc != PS_OK) {
      streams[dev] = nullptr;
      return nullptr;
    }
    owner[dev] = ctx;
  }
  return streams[dev];
}

// Runs between the window decode and the merge: fork the caller's stream (at the point
// recorded before the decode) onto the side stream, launch the prefix pass there, join.
struct PrefixFork {
  SharedPrefixLaunch sp;
  cudaEvent_t fork;
  cudaStream_t side;
};
int launch_prefix_forked(void* ctx, cudaStream_t stream) {
  PrefixFork* f = static_cast<PrefixFork*>(ctx);
  cudaEvent_t join = nullptr;
  int rc = check_cuda(cudaEventCreateWithFlags(&join, cudaEventDisableTiming), "cudaEventCreate");
  if (rc != PS_OK) return rc;
  rc = check_cuda(cudaStreamWaitEvent(f->side, f->fork, 0), "cudaStreamWaitEvent");
  if (rc == PS_OK) rc = launch_shared_prefix(f->sp, f->side);
  if (rc == PS_OK) rc = check_cuda(cudaEventRecord(join, f->side), "cudaEventRecord");
  if (rc == PS_OK) rc = check_cuda(cudaStreamWaitEvent(stream, join, 0), "cudaStreamWaitEvent");
  cudaEventDestroy(join);  // released once the recorded work completes
  return rc;
}
}  // namespace
}  // namespace ps

using namespace ps;

extern "C" {

const char* ps_last_error(void) { return g_last_error.c_str(); }

const char* ps_version(void) { return "libps 0.1 (sm_100a)"; }

int ps_kv_append_rope(const ps_params* params, const ps_kv_cache* cache, const void* k_new,
                      const void* v_new, void* q_inout, const int64_t* pos0, int32_t T,
                      int32_t* dev_status, ps_stream_t stream) {
  g_last_error.clear();
  PS_TRY(check_params(params, true));
  if (!cache) return fail(PS_ERR_INVALID_ARG, "cache is NULL");
  if (cache->batch < 0) return fail(PS_ERR_INVALID_ARG, "cache->batch must be >= 0");
  if (T < 1) return fail(PS_ERR_INVALID_ARG, "T must be >= 1");
  if (cache->batch == 0) return PS_OK;
  const bool linear = cache->k_ring == nullptr && cache->v_ring == nullptr;
  if (!linear) {
    PS_TRY(check_ptr(cache->k_ring, "cache->k_ring"));
    PS_TRY(check_ptr(cache->v_ring, "cache->v_ring"));
  }
  // a ring cache whose prefix pointers are both NULL is ring-only: tokens at positions
  // below l_prefix are skipped (their prefix rows live elsewhere)
  const bool ring_only = !linear && cache->k_prefix == nullptr && cache->v_prefix == nullptr;
  if ((params->l_prefix > 0 && !ring_only) || linear) {
    PS_TRY(check_ptr(cache->k_prefix, "cache->k_prefix"));
    PS_TRY(check_ptr(cache->v_prefix, "cache->v_prefix"));
  }
  if (linear && params->l_prefix < 1)
    return fail(PS_ERR_INVALID_ARG, "a linear cache (ring NULL) needs l_prefix = Lmax >= 1");
  PS_TRY(check_ptr(k_new, "k_new"));
  PS_TRY(check_ptr(v_new, "v_new"));
  PS_TRY(check_ptr(q_inout, "q_inout", true));
  if (!pos0) return fail(PS_ERR_INVALID_ARG, "pos0 is NULL");
  if ((reinterpret_cast<uintptr_t>(pos0) & 7u) != 0)
    return fail(PS_ERR_INVALID_ARG, "pos0 is not 8-byte aligned");
  if ((reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return fail(PS_ERR_INVALID_ARG, "dev_status is not 4-byte aligned");
  AppendArgs a{};
  a.k_new = k_new;
  a.v_new = v_new;
  a.q = q_inout;
  a.pos0 = pos0;
  a.k_pre = cache->k_prefix;
  a.v_pre = cache->v_prefix;
  a.k_ring = linear ? nullptr : cache->k_ring;
  a.v_ring = linear ? nullptr : cache->v_ring;
  a.status = dev_status;
  a.batch = cache->batch;
  a.T = T;
  a.hq = params->n_q_heads;
  a.hkv = params->n_kv_heads;
  a.lp = params->l_prefix;
  a.w = params->window;
  for (int i = 0; i < kHeadDim / 2; ++i)
    a.inv_freq[i] = pow(params->rope_theta, -2.0 * i / double(kHeadDim));
  return check_cuda(launch_append(a, reinterpret_cast<cudaStream_t>(stream)),
                    "append_rope_kernel launch");
}

size_t ps_decode_workspace_bytes(const ps_params* params, int64_t batch) {
  if (check_params(params, true) != PS_OK || batch < 0) return 0;
  return decode_workspace_bytes(batch, params->n_kv_heads,
                                (int64_t)params->l_prefix + params->window);
}

// Checks shared by every decode entry point over the contiguous store, and the launch
// description they build.  *empty is set (PS_OK returned) when there is nothing to launch.
static int decode_prepare(const ps_params* params, const ps_kv_cache* cache, const void* q,
                          const int64_t* pos, void* out, float* lse, int32_t* dev_status,
                          DecodeLaunch* l, bool* empty) {
  *empty = false;
  PS_TRY(check_params(params, true));
  if (params->n_q_heads / params->n_kv_heads > kMaxGroup)
    return fail(PS_ERR_UNSUPPORTED, "decode supports at most 8 query heads per KV head");
  if (!cache) return fail(PS_ERR_INVALID_ARG, "cache is NULL");
  if (cache->batch < 0) return fail(PS_ERR_INVALID_ARG, "cache->batch must be >= 0");
  if (cache->batch == 0) {
    *empty = true;
    return PS_OK;
  }
  PS_TRY(check_ptr(cache->k_ring, "cache->k_ring"));
  PS_TRY(check_ptr(cache->v_ring, "cache->v_ring"));
  if (params->l_prefix > 0) {
    PS_TRY(check_ptr(cache->k_prefix, "cache->k_prefix"));
    PS_TRY(check_ptr(cache->v_prefix, "cache->v_prefix"));
  }
  PS_TRY(check_ptr(q, "q"));
  PS_TRY(check_ptr(out, "out"));
  PS_TRY(check_ptr(lse, "lse", true));
  if (!pos) return fail(PS_ERR_INVALID_ARG, "pos is NULL");
  if ((reinterpret_cast<uintptr_t>(pos) & 7u) != 0)
    return fail(PS_ERR_INVALID_ARG, "pos is not 8-byte aligned");
  if ((reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return fail(PS_ERR_INVALID_ARG, "dev_status is not 4-byte aligned");
  *l = DecodeLaunch{};
  l->q = q;
  l->pos = pos;
  l->out = out;
  l->lse = lse;
  l->status = dev_status;
  l->batch = cache->batch;
  l->hq = params->n_q_heads;
  l->hkv = params->n_kv_heads;
  l->lp = params->l_prefix;
  l->w = params->window;
  l->lmax = 0;
  l->full_mode = 0;
  l->scale = resolve_scale(params);
  l->k0 = cache->k_prefix;
  l->v0 = cache->v_prefix;
  l->k1 = cache->k_ring;
  l->v1 = cache->v_ring;
  l->rope_theta = params->rope_theta;
  return PS_OK;
}

static int decode_entry(const ps_params* params, const ps_kv_cache* cache, const void* q,
                        const int64_t* pos, void* out, float* lse, void* workspace,
                        size_t ws_bytes, int32_t* dev_status, ps_stream_t stream,
                        int32_t reset_pe, int32_t lcap = 0, const int32_t* pin_count = nullptr,
                        const int64_t* pin_pos = nullptr, int32_t after_append = 0) {
  g_last_error.clear();
  DecodeLaunch l;
  bool empty = false;
  PS_TRY(decode_prepare(params, cache, q, pos, out, lse, dev_status, &l, &empty));
  if (empty) return PS_OK;
  const int64_t pre_rows = lcap > params->l_prefix ? lcap : params->l_prefix;
  const size_t need = decode_workspace_bytes(cache->batch, params->n_kv_heads,
                                             pre_rows + params->window);
  if (need > 0) {
    if (!workspace || ws_bytes < need)
      return fail(PS_ERR_WORKSPACE, "workspace smaller than the decode workspace size");
    PS_TRY(check_ptr(workspace, "workspace"));
  }
  l.workspace = workspace;
  l.reset_pe = reset_pe;
  l.lcap = lcap;
  l.pin_count = pin_count;
  l.pin_pos = pin_pos;
  l.after_append = after_append;
  return launch_decode(l, reinterpret_cast<cudaStream_t>(stream));
}

int ps_decode_attn(const ps_params* params, const ps_kv_cache* cache, const void* q,
                   const int64_t* pos, void* out, float* lse, void* workspace, size_t ws_bytes,
                   int32_t* dev_status, ps_stream_t stream) {
  return decode_entry(params, cache, q, pos, out, lse, workspace, ws_bytes, dev_status, stream,
                      0);
}

int ps_decode_attn_reset_pe(const ps_params* params, const ps_kv_cache* cache, const void* q,
                            const int64_t* pos, void* out, float* lse, void* workspace,
                            size_t ws_bytes, int32_t* dev_status, ps_stream_t stream) {
  return decode_entry(params, cache, q, pos, out, lse, workspace, ws_bytes, dev_status, stream,
                      1);
}

int ps_decode_attn_noalloc(const ps_params* params, const ps_kv_cache* cache, const void* q,
                           const int64_t* pos, void* out, float* lse, int32_t* dev_status,
                           ps_stream_t stream) {
  g_last_error.clear();
  DecodeLaunch l;
  bool empty = false;
  PS_TRY(decode_prepare(params, cache, q, pos, out, lse, dev_status, &l, &empty));
  if (empty) return PS_OK;
  return launch_decode_static_scratch(l, reinterpret_cast<cudaStream_t>(stream));
}

size_t ps_full_attn_workspace_bytes(const ps_params* params, int64_t batch, int64_t lmax) {
  if (check_params(params, false) != PS_OK || batch < 0 || lmax < 1) return 0;
  return decode_workspace_bytes(batch, params->n_kv_heads, lmax);
}

int ps_full_attn_ref(const ps_params* params, const void* k_full, const void* v_full,
                     int64_t lmax, const void* q, const int64_t* pos, int64_t batch, void* out,
                     float* lse, void* workspace, size_t ws_bytes, int32_t* dev_status,
                     ps_stream_t stream) {
  g_last_error.clear();
  PS_TRY(check_params(params, false));
  if (params->n_q_heads / params->n_kv_heads > kMaxGroup)
    return fail(PS_ERR_UNSUPPORTED, "decode supports at most 8 query heads per KV head");
  if (batch < 0) return fail(PS_ERR_INVALID_ARG, "batch must be >= 0");
  if (lmax < 1 || lmax > 0x7fffffffLL) return fail(PS_ERR_INVALID_ARG, "lmax out of range");
  if (batch == 0) return PS_OK;
  PS_TRY(check_ptr(k_full, "k_full"));
  PS_TRY(check_ptr(v_full, "v_full"));
  PS_TRY(check_ptr(q, "q"));
  PS_TRY(check_ptr(out, "out"));
  PS_TRY(check_ptr(lse, "lse", true));
  if (!pos) return fail(PS_ERR_INVALID_ARG, "pos is NULL");
  if ((reinterpret_cast<uintptr_t>(pos) & 7u) != 0)
    return fail(PS_ERR_INVALID_ARG, "pos is not 8-byte aligned");
  const size_t need = decode_workspace_bytes(batch, params->n_kv_heads, lmax);
  if (need > 0) {
    if (!workspace || ws_bytes < need)
      return fail(PS_ERR_WORKSPACE, "workspace smaller than ps_full_attn_workspace_bytes()");
    PS_TRY(check_ptr(workspace, "workspace"));
  }
  DecodeLaunch l{};
  l.q = q;
  l.pos = pos;
  l.out = out;
  l.lse = lse;
  l.workspace = workspace;
  l.status = dev_status;
  l.batch = batch;
  l.hq = params->n_q_heads;
  l.hkv = params->n_kv_heads;
  l.lp = 0;
  l.w = 1;
  l.lmax = lmax;
  l.full_mode = 1;
  l.scale = resolve_scale(params);
  l.k0 = k_full;
  l.v0 = v_full;
  l.k1 = nullptr;
  l.v1 = nullptr;
  return launch_decode(l, reinterpret_cast<cudaStream_t>(stream));
}

int ps_decode_visible_ranges(const ps_params* params, const int64_t* pos, int64_t batch,
                             int32_t* ranges_out, ps_stream_t stream) {
  g_last_error.clear();
  PS_TRY(check_params(params, true));
  if (batch < 0) return fail(PS_ERR_INVALID_ARG, "batch must be >= 0");
  if (batch == 0) return PS_OK;
  if (!pos || !ranges_out) return fail(PS_ERR_INVALID_ARG, "pos / ranges_out is NULL");
  return check_cuda(launch_visible_ranges(pos, batch, params->l_prefix, params->window,
                                          ranges_out, reinterpret_cast<cudaStream_t>(stream)),
                    "visible_ranges_kernel launch");
}

int ps_check_wait_timeout(int32_t* dev_status, ps_stream_t stream) {
  g_last_error.clear();
  if (!dev_status || (reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return fail(PS_ERR_INVALID_ARG, "dev_status is NULL or not 4-byte aligned");
  return check_cuda(launch_wait_timeout(dev_status, reinterpret_cast<cudaStream_t>(stream)),
                    "wait_timeout_kernel launch");
}

int ps_prefill_tile_geometry(int32_t* bq, int32_t* bk) {
  if (!bq || !bk) return fail(PS_ERR_INVALID_ARG, "bq / bk is NULL");
  *bq = kPrefillBq;
  *bk = kPrefillBk;
  return PS_OK;
}

int64_t ps_prefill_plan_tiles(const ps_params* params, int64_t seq) {
  if (check_params(params, true) != PS_OK) return PS_ERR_INVALID_ARG;
  if (seq < 1) return fail(PS_ERR_INVALID_ARG, "seq must be >= 1");
  return prefill_plan_tiles(seq, params->l_prefix, params->window);
}

size_t ps_prefill_workspace_bytes(const ps_params* params, int64_t batch, int64_t seq) {
  if (check_params(params, true) != PS_OK || batch < 0 || seq < 1) return 0;
  return prefill_workspace_bytes(seq, params->l_prefix, params->window);
}

int ps_masked_prefill_attn(const ps_params* params, const void* q, const void* k, const void* v,
                           int64_t batch, int64_t seq, void* out, float* lse, int32_t* tile_plan,
                           int64_t tile_plan_cap, int64_t* n_tiles, void* workspace,
                           size_t ws_bytes, int32_t* dev_status, ps_stream_t stream) {
  g_last_error.clear();
  PS_TRY(check_params(params, true));
  if (batch < 0) return fail(PS_ERR_INVALID_ARG, "batch must be >= 0");
  if (seq < 1 || seq > (1LL << 30)) return fail(PS_ERR_INVALID_ARG, "seq out of range");
  const int64_t nt = prefill_plan_tiles(seq, params->l_prefix, params->window);
  if (n_tiles) *n_tiles = nt;
  if (tile_plan) {
    PS_TRY(check_ptr(tile_plan, "tile_plan"));
    if (tile_plan_cap < nt) return fail(PS_ERR_INVALID_ARG, "tile_plan_cap smaller than the plan");
  }
  if (batch == 0) return PS_OK;
  PS_TRY(check_ptr(q, "q"));
  PS_TRY(check_ptr(k, "k"));
  PS_TRY(check_ptr(v, "v"));
  PS_TRY(check_ptr(out, "out"));
  PS_TRY(check_ptr(lse, "lse", true));
  if ((reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return fail(PS_ERR_INVALID_ARG, "dev_status is not 4-byte aligned");
  if (batch > 0x7fffffffLL) return fail(PS_ERR_UNSUPPORTED, "batch too large");
  const size_t need = prefill_workspace_bytes(seq, params->l_prefix, params->window);
  if (need > 0) {
    if (!workspace || ws_bytes < need)
      return fail(PS_ERR_WORKSPACE, "workspace smaller than ps_prefill_workspace_bytes()");
    PS_TRY(check_ptr(workspace, "workspace"));
  }
  PrefillLaunch l{};
  l.q = q;
  l.k = k;
  l.v = v;
  l.out = out;
  l.lse = lse;
  l.plan_out = tile_plan;
  l.workspace = workspace;
  l.batch = batch;
  l.seq = seq;
  l.hq = params->n_q_heads;
  l.hkv = params->n_kv_heads;
  l.lp = params->l_prefix;
  l.w = params->window;
  l.scale = resolve_scale(params);
  l.n_tiles = nt;
  l.status = dev_status;
  return launch_prefill(l, reinterpret_cast<cudaStream_t>(stream));
}

size_t ps_prefill_bwd_workspace_bytes(const ps_params* params, int64_t batch, int64_t seq) {
  if (check_params(params, true) != PS_OK || batch < 0 || seq < 1 || seq > (1LL << 30)) return 0;
  return prefill_bwd_workspace_bytes(batch, params->n_q_heads, seq, params->l_prefix,
                                     params->window);
}

int ps_masked_prefill_attn_bwd(const ps_params* params, const void* q, const void* k,
                               const void* v, const void* out, const void* dout,
                               const float* lse, int64_t batch, int64_t seq, void* dq, void* dk,
                               void* dv, void* workspace, size_t ws_bytes, int32_t* dev_status,
                               ps_stream_t stream) {
  g_last_error.clear();
  PS_TRY(check_params(params, true));
  if (batch < 0) return fail(PS_ERR_INVALID_ARG, "batch must be >= 0");
  if (seq < 1 || seq > (1LL << 30)) return fail(PS_ERR_INVALID_ARG, "seq out of range");
  if (batch == 0) return PS_OK;
  if (batch > 0x7fffffffLL) return fail(PS_ERR_UNSUPPORTED, "batch too large");
  PS_TRY(check_ptr(q, "q"));
  PS_TRY(check_ptr(k, "k"));
  PS_TRY(check_ptr(v, "v"));
  PS_TRY(check_ptr(out, "out"));
  PS_TRY(check_ptr(dout, "dout"));
  PS_TRY(check_ptr(lse, "lse"));
  PS_TRY(check_ptr(dq, "dq"));
  PS_TRY(check_ptr(dk, "dk"));
  PS_TRY(check_ptr(dv, "dv"));
  if ((reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return fail(PS_ERR_INVALID_ARG, "dev_status is not 4-byte aligned");
  // one sequence per pass at least; more per pass as the workspace allows
  const size_t need =
      prefill_bwd_min_workspace_bytes(params->n_q_heads, seq, params->l_prefix, params->window);
  if (!workspace || ws_bytes < need)
    return fail(PS_ERR_WORKSPACE, "workspace smaller than ps_prefill_bwd_workspace_bytes(batch 1)");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(PS_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  PrefillBwdLaunch l{};
  l.q = q;
  l.k = k;
  l.v = v;
  l.out = out;
  l.dout = dout;
  l.lse = lse;
  l.dq = dq;
  l.dk = dk;
  l.dv = dv;
  l.workspace = workspace;
  l.ws_bytes = ws_bytes;
  l.batch = batch;
  l.seq = seq;
  l.hq = params->n_q_heads;
  l.hkv = params->n_kv_heads;
  l.lp = params->l_prefix;
  l.w = params->window;
  l.scale = resolve_scale(params);
  l.status = dev_status;
  return launch_prefill_bwd(l, reinterpret_cast<cudaStream_t>(stream));
}

size_t ps_decode_shared_prefix_workspace_bytes(const ps_params* params, int64_t batch,
                                               int64_t group_size) {
  if (check_params(params, true) != PS_OK || batch < 0 || group_size < 1 ||
      batch % group_size != 0 || params->l_prefix < 1)
    return 0;
  return shared_prefix_layout(params, batch, group_size).total;
}

int ps_decode_attn_shared_prefix(const ps_params* params, const ps_kv_cache* cache,
                                 int64_t group_size, const void* q, const int64_t* pos,
                                 void* out, float* lse, void* workspace, size_t ws_bytes,
                                 int32_t* dev_status, ps_stream_t stream) {
  g_last_error.clear();
  PS_TRY(check_params(params, true));
  if (params->n_q_heads / params->n_kv_heads > kMaxGroup)
    return fail(PS_ERR_UNSUPPORTED, "decode supports at most 8 query heads per KV head");
  if (params->l_prefix < 1)
    return fail(PS_ERR_INVALID_ARG, "shared-prefix decode needs l_prefix >= 1");
  if (!cache) return fail(PS_ERR_INVALID_ARG, "cache is NULL");
  if (cache->batch < 0) return fail(PS_ERR_INVALID_ARG, "cache->batch must be >= 0");
  if (group_size < 1) return fail(PS_ERR_INVALID_ARG, "group_size must be >= 1");
  if (cache->batch % group_size != 0)
    return fail(PS_ERR_INVALID_ARG, "batch must be a multiple of group_size");
  if (cache->batch == 0) return PS_OK;
  if (group_size * (params->n_q_heads / params->n_kv_heads) > 0x7fffffffLL)
    return fail(PS_ERR_UNSUPPORTED, "group_size too large");
  PS_TRY(check_ptr(cache->k_ring, "cache->k_ring"));
  PS_TRY(check_ptr(cache->v_ring, "cache->v_ring"));
  PS_TRY(check_ptr(cache->k_prefix, "cache->k_prefix"));
  PS_TRY(check_ptr(cache->v_prefix, "cache->v_prefix"));
  PS_TRY(check_ptr(q, "q"));
  PS_TRY(check_ptr(out, "out"));
  PS_TRY(check_ptr(lse, "lse", true));
  if (!pos) return fail(PS_ERR_INVALID_ARG, "pos is NULL");
  if ((reinterpret_cast<uintptr_t>(pos) & 7u) != 0)
    return fail(PS_ERR_INVALID_ARG, "pos is not 8-byte aligned");
  if ((reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return fail(PS_ERR_INVALID_ARG, "dev_status is not 4-byte aligned");
  const SharedPrefixLayout L = shared_prefix_layout(params, cache->batch, group_size);
  if (!workspace || ws_bytes < L.total)
    return fail(PS_ERR_WORKSPACE, "workspace smaller than ps_decode_shared_prefix_workspace_bytes()");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(PS_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  char* ws = static_cast<char*>(workspace);
  float* o_pre = reinterpret_cast<float*>(ws + L.dec);
  float* lse2_pre = reinterpret_cast<float*>(ws + L.dec + L.o);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  SharedPrefixLaunch sp{};
  sp.q = q;
  sp.pos = pos;
  sp.k_pre = cache->k_prefix;
  sp.v_pre = cache->v_prefix;
  sp.o_pre = o_pre;
  sp.lse2_pre = lse2_pre;
  sp.status = dev_status;
  sp.batch = cache->batch;
  sp.gsize = group_size;
  sp.hq = params->n_q_heads;
  sp.hkv = params->n_kv_heads;
  sp.lp = params->l_prefix;
  sp.scale = resolve_scale(params);
  int rc = PS_OK;
  PrefixFork fk;
  fk.sp = sp;
  fk.side = side_stream(&rc);
  if (rc != PS_OK) return rc;
  rc = check_cuda(cudaEventCreateWithFlags(&fk.fork, cudaEventDisableTiming), "cudaEventCreate");
  if (rc != PS_OK) return rc;
  // the prefix pass may start as soon as the work queued so far on `stream` is done; it is
  // launched after the window decode, so that decode is first in line for the SMs
  rc = check_cuda(cudaEventRecord(fk.fork, st), "cudaEventRecord");
  if (rc != PS_OK) {
    cudaEventDestroy(fk.fork);
    return rc;
  }
  DecodeLaunch l{};
  l.q = q;
  l.pos = pos;
  l.out = out;
  l.lse = lse;
  l.workspace = workspace;  // the window pass's split-K partials come first (L.dec bytes)
  l.status = dev_status;
  l.batch = cache->batch;
  l.hq = params->n_q_heads;
  l.hkv = params->n_kv_heads;
  l.lp = params->l_prefix;
  l.w = params->window;
  l.scale = resolve_scale(params);
  l.k0 = cache->k_prefix;
  l.v0 = cache->v_prefix;
  l.k1 = cache->k_ring;
  l.v1 = cache->v_ring;
  l.skip_prefix = 1;
  l.pre_o = o_pre;
  l.pre_lse2 = lse2_pre;
  l.pre_splits = L.splits;
  l.before_merge = launch_prefix_forked;
  l.before_merge_ctx = &fk;
  rc = launch_decode(l, st);
  cudaEventDestroy(fk.fork);
  return rc;
}

int ps_kv_pin(const ps_params* params, const ps_kv_cache* cache, int32_t prefix_capacity,
              int32_t* pin_count, int64_t* pin_pos, const int64_t* t0, const int64_t* t1,
              const int64_t* pos, int32_t* dev_status, ps_stream_t stream) {
  g_last_error.clear();
  PS_TRY(check_params(params, true));
  if (!cache) return fail(PS_ERR_INVALID_ARG, "cache is NULL");
  if (cache->batch < 0) return fail(PS_ERR_INVALID_ARG, "cache->batch must be >= 0");
  if (prefix_capacity <= params->l_prefix)
    return fail(PS_ERR_INVALID_ARG, "prefix_capacity must exceed l_prefix");
  if (cache->batch == 0) return PS_OK;
  PS_TRY(check_ptr(cache->k_prefix, "cache->k_prefix"));
  PS_TRY(check_ptr(cache->v_prefix, "cache->v_prefix"));
  PS_TRY(check_ptr(cache->k_ring, "cache->k_ring"));
  PS_TRY(check_ptr(cache->v_ring, "cache->v_ring"));
  if (!pin_count || !pin_pos || !t0 || !t1 || !pos)
    return fail(PS_ERR_INVALID_ARG, "pin_count, pin_pos, t0, t1 and pos are required");
  if (((reinterpret_cast<uintptr_t>(pin_pos) | reinterpret_cast<uintptr_t>(t0) |
        reinterpret_cast<uintptr_t>(t1) | reinterpret_cast<uintptr_t>(pos)) & 7u) != 0 ||
      (reinterpret_cast<uintptr_t>(pin_count) & 3u) != 0)
    return fail(PS_ERR_INVALID_ARG, "misaligned pin metadata or positions");
  if ((reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return fail(PS_ERR_INVALID_ARG, "dev_status is not 4-byte aligned");
  PinArgs a;
  a.k_ring = cache->k_ring;
  a.v_ring = cache->v_ring;
  a.k_pre = cache->k_prefix;
  a.v_pre = cache->v_prefix;
  a.pin_count = pin_count;
  a.pin_pos = pin_pos;
  a.t0 = t0;
  a.t1 = t1;
  a.pos = pos;
  a.status = dev_status;
  a.batch = cache->batch;
  a.hkv = params->n_kv_heads;
  a.lp = params->l_prefix;
  a.w = params->window;
  a.lcap = prefix_capacity;
  return check_cuda(launch_pin(a, reinterpret_cast<cudaStream_t>(stream)), "pin_kernel launch");
}

size_t ps_decode_pinned_workspace_bytes(const ps_params* params, int64_t batch,
                                        int32_t prefix_capacity) {
  if (check_params(params, true) != PS_OK || batch < 0 || prefix_capacity < params->l_prefix)
    return 0;
  return decode_workspace_bytes(batch, params->n_kv_heads,
                                (int64_t)prefix_capacity + params->window);
}

int ps_decode_attn_pinned(const ps_params* params, const ps_kv_cache* cache,
                          int32_t prefix_capacity, const int32_t* pin_count,
                          const int64_t* pin_pos, const void* q, const int64_t* pos, void* out,
                          float* lse, void* workspace, size_t ws_bytes, int32_t* dev_status,
                          ps_stream_t stream) {
  g_last_error.clear();
  if (!params) return fail(PS_ERR_INVALID_ARG, "params is NULL");
  if (prefix_capacity <= params->l_prefix)
    return fail(PS_ERR_INVALID_ARG, "prefix_capacity must exceed l_prefix");
  if (!pin_count || !pin_pos) return fail(PS_ERR_INVALID_ARG, "pin_count and pin_pos required");
  if ((reinterpret_cast<uintptr_t>(pin_pos) & 7u) != 0 ||
      (reinterpret_cast<uintptr_t>(pin_count) & 3u) != 0)
    return fail(PS_ERR_INVALID_ARG, "misaligned pin metadata");
  return decode_entry(params, cache, q, pos, out, lse, workspace, ws_bytes, dev_status, stream,
                      0, prefix_capacity, pin_count, pin_pos);
}

int ps_decode_step(const ps_params* params, const ps_kv_cache* cache, const void* k_new,
                   const void* v_new, void* q_inout, const int64_t* pos, void* out, float* lse,
                   void* workspace, size_t ws_bytes, int32_t* dev_status, ps_stream_t stream) {
  g_last_error.clear();
  PS_TRY(check_ptr(q_inout, "q_inout"));
  // validate the decode half first, so that nothing is launched on a bad call
  if (!params) return fail(PS_ERR_INVALID_ARG, "params is NULL");
  PS_TRY(check_params(params, true));
  if (params->n_q_heads / params->n_kv_heads > kMaxGroup)
    return fail(PS_ERR_UNSUPPORTED, "decode supports at most 8 query heads per KV head");
  if (!cache) return fail(PS_ERR_INVALID_ARG, "cache is NULL");
  if (cache->batch > 0 && cache->k_ring == nullptr)
    return fail(PS_ERR_INVALID_ARG, "ps_decode_step needs a ring cache");
  const size_t need = decode_workspace_bytes(cache->batch, params->n_kv_heads,
                                             (int64_t)params->l_prefix + params->window);
  if (need > 0 && (!workspace || ws_bytes < need))
    return fail(PS_ERR_WORKSPACE, "workspace smaller than ps_decode_workspace_bytes()");
  PS_TRY(ps_kv_append_rope(params, cache, k_new, v_new, q_inout, pos, 1, dev_status, stream));
  return decode_entry(params, cache, q_inout, pos, out, lse, workspace, ws_bytes, dev_status,
                      stream, 0, 0, nullptr, nullptr, 1);
}

// ---------------------------------------------------------------- paged store
static int check_paged(const ps_params* params, const void* k_pool, const void* v_pool,
                       int64_t n_blocks, const int32_t* block_table, int32_t table_stride,
                       int64_t batch) {
  PS_TRY(check_params(params, true));
  if (params->window % kDecodeTile != 0)
    return fail(PS_ERR_UNSUPPORTED, "a paged store needs a window that is a multiple of 64");
  if (batch < 0) return fail(PS_ERR_INVALID_ARG, "batch must be >= 0");
  if (n_blocks < 1 || n_blocks > 0x7fffffffLL)
    return fail(PS_ERR_INVALID_ARG, "n_blocks out of range");
  const int32_t need = (params->l_prefix + kDecodeTile - 1) / kDecodeTile +
                       params->window / kDecodeTile;
  if (table_stride < need)
    return fail(PS_ERR_INVALID_ARG, "table_stride smaller than the blocks a sequence needs");
  PS_TRY(check_ptr(k_pool, "k_pool"));
  PS_TRY(check_ptr(v_pool, "v_pool"));
  if (!block_table || (reinterpret_cast<uintptr_t>(block_table) & 3u) != 0)
    return fail(PS_ERR_INVALID_ARG, "block_table is NULL or not 4-byte aligned");
  return PS_OK;
}

int ps_kv_append_rope_paged(const ps_params* params, void* k_pool, void* v_pool,
                            int64_t n_blocks, const int32_t* block_table, int32_t table_stride,
                            int64_t batch, const void* k_new, const void* v_new, void* q_inout,
                            const int64_t* pos0, int32_t T, int32_t* dev_status,
                            ps_stream_t stream) {
  g_last_error.clear();
  PS_TRY(check_paged(params, k_pool, v_pool, n_blocks, block_table, table_stride, batch));
  if (T < 1) return fail(PS_ERR_INVALID_ARG, "T must be >= 1");
  if (batch == 0) return PS_OK;
  PS_TRY(check_ptr(k_new, "k_new"));
  PS_TRY(check_ptr(v_new, "v_new"));
  PS_TRY(check_ptr(q_inout, "q_inout", true));
  if (!pos0 || (reinterpret_cast<uintptr_t>(pos0) & 7u) != 0)
    return fail(PS_ERR_INVALID_ARG, "pos0 is NULL or not 8-byte aligned");
  if ((reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return fail(PS_ERR_INVALID_ARG, "dev_status is not 4-byte aligned");
  AppendArgs a{};
  a.k_new = k_new;
  a.v_new = v_new;
  a.q = q_inout;
  a.pos0 = pos0;
  a.k_pre = k_pool;
  a.v_pre = v_pool;
  a.k_ring = k_pool;
  a.v_ring = v_pool;
  a.status = dev_status;
  a.batch = batch;
  a.T = T;
  a.hq = params->n_q_heads;
  a.hkv = params->n_kv_heads;
  a.lp = params->l_prefix;
  a.w = params->window;
  a.paged = 1;
  a.table = block_table;
  a.table_stride = table_stride;
  a.pre_blocks = (params->l_prefix + kDecodeTile - 1) / kDecodeTile;
  a.n_blocks = n_blocks;
  for (int i = 0; i < kHeadDim / 2; ++i)
    a.inv_freq[i] = pow(params->rope_theta, -2.0 * i / double(kHeadDim));
  return check_cuda(launch_append(a, reinterpret_cast<cudaStream_t>(stream)),
                    "append_rope_kernel launch");
}

int ps_decode_attn_paged(const ps_params* params, void* k_pool, void* v_pool, int64_t n_blocks,
                         const int32_t* block_table, int32_t table_stride, int64_t batch,
                         const void* q, const int64_t* pos, void* out, float* lse,
                         void* workspace, size_t ws_bytes, int32_t* dev_status,
                         ps_stream_t stream) {
  g_last_error.clear();
  PS_TRY(check_paged(params, k_pool, v_pool, n_blocks, block_table, table_stride, batch));
  if (params->n_q_heads / params->n_kv_heads > kMaxGroup)
    return fail(PS_ERR_UNSUPPORTED, "decode supports at most 8 query heads per KV head");
  if (batch == 0) return PS_OK;
  PS_TRY(check_ptr(q, "q"));
  PS_TRY(check_ptr(out, "out"));
  PS_TRY(check_ptr(lse, "lse", true));
  if (!pos || (reinterpret_cast<uintptr_t>(pos) & 7u) != 0)
    return fail(PS_ERR_INVALID_ARG, "pos is NULL or not 8-byte aligned");
  if ((reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return fail(PS_ERR_INVALID_ARG, "dev_status is not 4-byte aligned");
  const size_t need = decode_workspace_bytes(batch, params->n_kv_heads,
                                             (int64_t)params->l_prefix + params->window);
  if (need > 0 && (!workspace || ws_bytes < need))
    return fail(PS_ERR_WORKSPACE, "workspace smaller than ps_decode_workspace_bytes()");
  DecodeLaunch l{};
  l.q = q;
  l.pos = pos;
  l.out = out;
  l.lse = lse;
  l.workspace = workspace;
  l.status = dev_status;
  l.batch = batch;
  l.hq = params->n_q_heads;
  l.hkv = params->n_kv_heads;
  l.lp = params->l_prefix;
  l.w = params->window;
  l.scale = resolve_scale(params);
  l.k0 = k_pool;
  l.v0 = v_pool;
  l.k1 = k_pool;
  l.v1 = v_pool;
  l.rope_theta = params->rope_theta;
  l.paged = 1;
  l.table = block_table;
  l.table_stride = table_stride;
  l.n_blocks = n_blocks;
  return launch_decode(l, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
