// Internal declarations shared by the libps translation units (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <utility>

#include "../../include/ps.h"

namespace ps {

constexpr int kHeadDim = 128;
constexpr int kMaxGroup = 8;  // query heads per KV head handled by one decode CTA

// Records a host-side failure message for ps_last_error() and returns `code`.
int fail(int code, const std::string& msg);
// Maps a CUDA runtime error to PS_ERR_CUDA with its message (PS_OK if no error).
int check_cuda(cudaError_t e, const char* what);

// Encodes a 3-D bf16 tensor map [z][y][x] with a box of {box_x, box_y, 1} and 128-byte
// swizzle.  Returns false (with a message recorded) on failure.
bool make_map_3d(CUtensorMap* map, const void* base, uint64_t x, uint64_t y, uint64_t z,
                 uint32_t box_x, uint32_t box_y);

// Encodes a 4-D bf16 tensor map (dims innermost first, dense strides) with 128-byte swizzle.
bool make_map_4d(CUtensorMap* map, const void* base, const uint64_t dims[4],
                 const uint32_t box[4]);

// Launches `kernel` with programmatic stream serialization: it may begin while the previous
// kernel of the stream finishes, and must call pdl_wait() before touching data that kernel
// (or anything before it) produced.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Streaming multiprocessor count of the current device.
int sm_count();

// ---------------------------------------------------------------- append
struct AppendArgs {
  const void* k_new;
  const void* v_new;
  void* q;
  const int64_t* pos0;
  void* k_pre;
  void* v_pre;
  void* k_ring;
  void* v_ring;
  int32_t* status;
  int64_t batch;
  int32_t T, hq, hkv, lp, w;
  // paged store: k_pre/v_pre and k_ring/v_ring all point to the pool [n_blocks][Hkv][64][D];
  // position p lives in logical block p / 64 (prefix) or pre_blocks + slot / 64 (ring) of
  // table[b * table_stride + ...]
  int32_t paged;
  const int32_t* table;
  int32_t table_stride, pre_blocks;
  int64_t n_blocks;
  double inv_freq[kHeadDim / 2];  // theta^(-2i/D), float64, filled by the host
};
cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);

// Appends tokens [t0[b], t1[b]) of each sequence, still in its window, to its pinned
// prefix: copies their (already rotated) K/V rows from the ring into prefix rows
// [lp + pin_count[b], ...) of a store with lcap rows and records their positions.
struct PinArgs {
  const void* k_ring;
  const void* v_ring;
  void* k_pre;
  void* v_pre;
  int32_t* pin_count;
  int64_t* pin_pos;
  const int64_t* t0;
  const int64_t* t1;
  const int64_t* pos;
  int32_t* status;
  int64_t batch;
  int32_t hkv, lp, w, lcap;
};
cudaError_t launch_pin(const PinArgs& a, cudaStream_t stream);

// ---------------------------------------------------------------- decode
struct DecodeLaunch {
  const void* q;
  const int64_t* pos;
  void* out;
  float* lse;
  void* workspace;
  int32_t* status;
  int64_t batch;
  int32_t hq, hkv;
  int32_t lp, w;
  int64_t lmax;        // full-attention mode: rows of the linear cache
  int32_t full_mode;   // 1: attend [0, pos] of a linear cache
  float scale;
  const void *k0, *v0;  // prefix (or linear) cache
  const void *k1, *v1;  // ring (unused in full mode)
  // Shared-prefix decode: read only the window (the prefix rows are skipped); the split-K
  // merge folds in precomputed prefix partials per (sequence, query head): normalised fp32
  // o and its base-2 lse (scores scaled by scale * log2 e).  Forces the stream-K schedule.
  int32_t skip_prefix;
  const float* pre_o;     // [pre_splits][batch, Hq, D]
  const float* pre_lse2;  // [pre_splits][batch, Hq]
  int32_t pre_splits;     // partials per (sequence, query head), each over a key range
  // called after the decode kernel is launched and before the merge (e.g. to launch the
  // prefix pass on another stream and make `stream` wait for it); PS_OK to continue
  int (*before_merge)(void* ctx, cudaStream_t stream);
  void* before_merge_ctx;
  // Reset PE (window renumbered after the prefix): prefix tiles use the query rotated at its
  // Reset-PE id L_prefix + |window| - 1 instead of its absolute position
  int32_t reset_pe;
  double rope_theta;
  // prefix store with room for tokens appended at run time: lcap rows per (sequence, KV
  // head); rows [lp, lp + pin_count[b]) hold promoted positions pin_pos[b][..] (ascending)
  int32_t lcap;
  const int32_t* pin_count;
  const int64_t* pin_pos;
  // the previous kernel on the stream is the one-token append at pos (ps_decode_step)
  int32_t after_append;
  // paged store (k0/v0 = the pool [n_blocks][Hkv][64][D], table [batch][table_stride])
  int32_t paged;
  const int32_t* table;
  int32_t table_stride;
  int64_t n_blocks;
};
// Split count and workspace bytes for a decode of this shape on the current device.
int decode_splits(int64_t batch, int32_t hkv, int64_t max_keys);
size_t decode_workspace_bytes(int64_t batch, int32_t hkv, int64_t max_keys,
                              bool force_streamk = false);
int launch_decode(const DecodeLaunch& a, cudaStream_t stream);
// Shared-prefix pass: attention of every (sequence, query head) of a group of `gsize`
// sequences over the group's prefix rows [0, min(pos + 1, lp)); writes o_pre/lse2_pre.
struct SharedPrefixLaunch {
  const void* q;         // [batch, Hq, D]
  const int64_t* pos;    // [batch]
  const void* k_pre;     // [batch / gsize, Hkv, lp, D]
  const void* v_pre;
  float* o_pre;          // [splits][batch, Hq, D]
  float* lse2_pre;       // [splits][batch, Hq]
  int32_t* status;
  int64_t batch, gsize;
  int32_t hq, hkv, lp;
  float scale;
};
// Key-range splits of the shared-prefix pass (enough CTAs to cover the SMs).
int shared_prefix_splits(int64_t batch, int64_t gsize, int32_t hq, int32_t hkv, int32_t lp);
int launch_shared_prefix(const SharedPrefixLaunch& l, cudaStream_t stream);
// Decode whose split-K scratch is the library's file-scope device array (no allocation).
constexpr size_t kDecodeScratchBytes = size_t(4) << 20;
int launch_decode_static_scratch(const DecodeLaunch& a, cudaStream_t stream);
cudaError_t launch_visible_ranges(const int64_t* pos, int64_t batch, int32_t lp, int32_t w,
                                  int32_t* out, cudaStream_t stream);

// ---------------------------------------------------------------- prefill
constexpr int kPrefillBq = 128;
constexpr int kPrefillBk = 128;
struct PrefillLaunch {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;
  int32_t* plan_out;  // optional copy of the plan
  void* workspace;
  int64_t batch, seq;
  int32_t hq, hkv, lp, w;
  float scale;
  int64_t n_tiles;  // plan rows per (batch, head)
  int32_t* status;
};
size_t prefill_workspace_bytes(int64_t seq, int32_t lp, int32_t w);
size_t prefill_plan_bytes(int64_t seq, int64_t n_tiles);
cudaError_t launch_plan(int64_t seq, int32_t lp, int32_t w, int64_t n_tiles, void* workspace,
                        int32_t* plan_out, cudaStream_t stream);
int64_t prefill_plan_tiles(int64_t seq, int32_t lp, int32_t w);
int launch_prefill(const PrefillLaunch& a, cudaStream_t stream);

// ---------------------------------------------------------------- prefill backward
struct PrefillBwdLaunch {
  const void* q;
  const void* k;
  const void* v;
  const void* out;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  void* workspace;
  size_t ws_bytes;  // sequences run in passes of as many as this workspace holds
  int64_t batch, seq;
  int32_t hq, hkv, lp, w;
  float scale;
  int32_t* status;
};
// Recommended workspace: the whole batch in one pass, unless its dS^T store would pass 4 GiB
// (then passes of fewer sequences).  The minimum holds one sequence.
size_t prefill_bwd_workspace_bytes(int64_t batch, int32_t hq, int64_t seq, int32_t lp, int32_t w);
size_t prefill_bwd_min_workspace_bytes(int32_t hq, int64_t seq, int32_t lp, int32_t w);
int launch_prefill_bwd(const PrefillBwdLaunch& l, cudaStream_t stream);

}  // namespace ps
