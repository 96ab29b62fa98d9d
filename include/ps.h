/*
 * ps.h -- C ABI of libps.so, the Prefix Sliding attention hot path for NVIDIA B200 (sm_100a).
 *
 * Prefix Sliding ("Prefix Sliding 完全拆解", pinghaoyang blog, §核心机制, eq. A(i)): the
 * query at (1-indexed) position i may attend key j iff j <= L_prefix or i - W < j <= i.
 * Every other key is evicted.  At most L_prefix + W keys are visible (same section,
 * eq. L_total), so decode cost per token is constant once the window is full.
 *
 * This library uses 0-based absolute positions.  The query at position p sees
 *     V(p) = { k : 0 <= k <= p  and  (k < l_prefix  or  k > p - window) }.
 * The window holds the W positions ending at, and including, the query.
 *
 * Conventions for every call:
 *   - The caller owns every buffer.  The library never allocates, frees or synchronises.
 *     Every call is asynchronous on the given stream.
 *   - "device" pointers live in GPU global memory; "host" pointers in CPU memory.
 *   - bf16 = IEEE bfloat16 stored as uint16.  All device buffers must be 16-byte aligned.
 *   - Host-detectable problems (null pointer, unsupported shape, n_q_heads % n_kv_heads
 *     != 0, workspace too small, misaligned pointer) return a negative ps_status and
 *     launch nothing.  ps_last_error() then describes the failure.
 *   - Conditions only the device can see (a position < 0, or past the end of a linear
 *     cache) set a bit in the optional device word *dev_status (atomic OR).  The kernel
 *     then skips that sequence: its output rows are written as zeros and its lse as
 *     -inf.  No kernel traps.
 *   - Every wait inside a kernel is bounded (about one second).  A wait that runs out
 *     sets PS_DEV_TIMEOUT in *dev_status and the kernel returns.
 */
#ifndef PS_H_
#define PS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so callers need no CUDA headers.
 * NULL selects the legacy default stream. */
typedef struct CUstream_st* ps_stream_t;

typedef enum {
  PS_OK = 0,
  PS_ERR_INVALID_ARG = -1, /* null pointer, bad size, misaligned pointer            */
  PS_ERR_UNSUPPORTED = -2, /* shape outside what the library implements              */
  PS_ERR_WORKSPACE = -3,   /* workspace null or smaller than the *_workspace_bytes  */
  PS_ERR_CUDA = -4         /* a CUDA runtime call or kernel launch failed           */
} ps_status;

/* Bits of *dev_status (device int32, OR-ed by kernels; the caller clears it). */
#define PS_DEV_BAD_POS 1   /* a position < 0: that sequence was skipped            */
#define PS_DEV_POS_RANGE 2 /* a position past the end of a linear (full) cache      */
#define PS_DEV_TIMEOUT 4   /* a bounded in-kernel wait ran out; output is invalid   */

/* Tile flags of the prefill plan ("Prefix Sliding 完全拆解", §Kernel 实现, two-level
 * filtering: SKIP tiles are neither loaded nor computed and never appear in a plan;
 * PARTIAL tiles get an element-wise mask; FULL tiles need none). */
#define PS_TILE_FULL 1
#define PS_TILE_PARTIAL 2

/* Attention geometry, shared by every call. */
typedef struct {
  int32_t n_q_heads;   /* Hq; Hq % Hkv == 0                                          */
  int32_t n_kv_heads;  /* Hkv; GQA: query head h reads KV head h / (Hq / Hkv)        */
  int32_t head_dim;    /* D; the library supports D == 128 only                       */
  int32_t l_prefix;    /* L_prefix >= 0; 0 gives the pure sliding window            */
  int32_t window;      /* W >= 1                                                    */
  int32_t reserved;    /* must be 0                                                 */
  double rope_theta;   /* RoPE base (rotate-half form), e.g. 1e6; > 0               */
  float softmax_scale; /* 0 selects 1/sqrt(head_dim)                                 */
  int32_t reserved2;   /* must be 0                                                 */
} ps_params;

/* Per-sequence bounded KV store: a pinned prefix region plus a W-slot ring.
 * Position p < l_prefix lives in prefix row p; position p >= l_prefix lives in ring slot
 * (p - l_prefix) mod W.  Writing a slot evicts the position it held (hard eviction,
 * §核心机制); cached keys are never rotated again (Continue PE, §位置编码).
 * Layouts (device, bf16, contiguous):
 *   k_prefix, v_prefix : [batch, Hkv, l_prefix, D]   (may be NULL when l_prefix == 0)
 *   k_ring,   v_ring   : [batch, Hkv, W, D]
 * A linear full-attention cache is the same struct with l_prefix = Lmax, window = 1 and
 * the ring pointers NULL; every position must then be < Lmax.
 * A ring-only cache has both prefix pointers NULL (and the ring set): ps_kv_append_rope then
 * writes only ring slots and skips tokens below l_prefix (PS_DEV_POS_RANGE); the prefix rows
 * live elsewhere, e.g. shared by a group of sequences (ps_decode_attn_shared_prefix). */
typedef struct {
  void* k_prefix;
  void* v_prefix;
  void* k_ring;
  void* v_ring;
  int64_t batch;
} ps_kv_cache;

/* Append T tokens per sequence and apply Continue-PE RoPE exactly once.
 * Source: §位置编码 (Continue PE: absolute position ids, rotated K reused as cached),
 * §核心机制 (hard eviction, bounded per-sequence store).
 *   k_new, v_new : device bf16 [batch, T, Hkv, D], raw (un-rotated) keys and values.
 *   q_inout      : device bf16 [batch, T, Hq, D] or NULL; rotated in place when given.
 *   pos0         : device int64 [batch]; token t of sequence b has absolute position
 *                  pos0[b] + t.  RoPE angles are position * theta^(-2i/D), formed and
 *                  reduced in float64.
 *   T            : tokens per sequence, >= 1.
 * When several of the T tokens map to one ring slot, only the latest is written (only
 * the last W positions beyond the prefix survive).  A token whose position is < 0 is
 * skipped (PS_DEV_BAD_POS); in a linear cache (ring NULL) a position >= l_prefix is
 * skipped (PS_DEV_POS_RANGE).  Its q rows are left as they were. */
int ps_kv_append_rope(const ps_params* params, const ps_kv_cache* cache, const void* k_new,
                      const void* v_new, void* q_inout, const int64_t* pos0, int32_t T,
                      int32_t* dev_status, ps_stream_t stream);

/* Bytes of device workspace ps_decode_attn needs for this geometry and batch (split-K
 * partial outputs).  Returns 0 on invalid arguments. */
size_t ps_decode_workspace_bytes(const ps_params* params, int64_t batch);

/* One decode step: attention of one query token per sequence over its visible keys.
 * Source: eq. A(i) and eq. L_total (§核心机制); §Kernel 实现 (only prefix and window
 * ranges are read; everything else is skipped).
 *   q     : device bf16 [batch, Hq, D], already rotated at pos[b] (ps_kv_append_rope).
 *   pos   : device int64 [batch], absolute position of the query; its own K/V must
 *           already be in the cache (append first, then decode).
 *   out   : device bf16 [batch, Hq, D].
 *   lse   : device fp32 [batch, Hq] or NULL; natural-log softmax denominator
 *           (max included) of scores q.k * scale.
 *   workspace, ws_bytes : device scratch of at least ps_decode_workspace_bytes(); its
 *           contents on entry do not matter.
 * Requires 1 <= Hq / Hkv <= 8. */
int ps_decode_attn(const ps_params* params, const ps_kv_cache* cache, const void* q,
                   const int64_t* pos, void* out, float* lse, void* workspace, size_t ws_bytes,
                   int32_t* dev_status, ps_stream_t stream);

/* One whole decode step: ps_kv_append_rope of one token per sequence at pos[b] (q rotated
 * in place), then ps_decode_attn at the same pos.  Source: §核心机制 and §位置编码 (append
 * with Continue PE, then attend the visible keys).  Results equal the two calls made one
 * after the other; because the library knows the append wrote exactly the newest row of
 * every sequence, the decode streams every other key tile while the append is still
 * running and waits for it only before that row and q.
 *   k_new, v_new : device bf16 [batch, Hkv, D], raw keys and values of the new token.
 *   q_inout      : device bf16 [batch, Hq, D], raw query; rotated at pos in place.
 * Other arguments, errors and the workspace (ps_decode_workspace_bytes) as ps_decode_attn;
 * a linear cache (ring NULL) is not accepted. */
int ps_decode_step(const ps_params* params, const ps_kv_cache* cache, const void* k_new,
                   const void* v_new, void* q_inout, const int64_t* pos, void* out, float* lse,
                   void* workspace, size_t ws_bytes, int32_t* dev_status, ps_stream_t stream);

/* One decode step under Reset PE, from the same Continue-PE cache ps_kv_append_rope fills.
 * Source: §位置编码 of "Prefix Sliding 完全拆解": Reset PE renumbers the window so that it
 * directly follows the prefix (the first window token gets id L_prefix, the next
 * L_prefix + 1, ...; the query, the newest window token, the last id); prefix ids are kept.
 * RoPE scores depend only on id differences, so against window keys these scores equal the
 * Continue-PE ones, and against prefix keys they equal Continue PE with the query rotated at
 * L_prefix + |window| - 1 instead of pos.  The kernel derives that second query from q (a
 * further rotation by L_prefix + |window| - 1 - pos, angles reduced in float64) and uses it
 * for the prefix rows; nothing in the cache is rotated again.  During warm-up (nothing
 * evicted) and with l_prefix = 0 the result equals ps_decode_attn.
 * Arguments, workspace (ps_decode_workspace_bytes), results and errors as ps_decode_attn;
 * q is rotated at pos (ps_kv_append_rope), as for ps_decode_attn. */
int ps_decode_attn_reset_pe(const ps_params* params, const ps_kv_cache* cache, const void* q,
                            const int64_t* pos, void* out, float* lse, void* workspace,
                            size_t ws_bytes, int32_t* dev_status, ps_stream_t stream);

/* ps_decode_attn without a workspace argument, for callers that cannot allocate device
 * memory: for example a plugin that its host framework hands only the input and output
 * buffers, or a fixed-memory serving loop where a cudaMalloc (or a caching allocator
 * growing) is not allowed between steps.  The paper has no counterpart; this is a
 * convenience of this library.
 * The split-K scratch lives in a device array built into libps (4 MiB = 4194304 bytes,
 * held on every GPU that loads the library until the process exits).  A shape whose
 * ps_decode_workspace_bytes() exceeds that returns PS_ERR_WORKSPACE and launches nothing.
 * This call never allocates or frees memory (no cudaMalloc, no cudaFree).  A call made outside
 * a stream capture looks up the array's device address with cudaGetSymbolAddress (with the
 * device current), so a context torn down and made again is never given a stale address; a
 * call inside a capture reuses the address the last call outside one found.  Make the first
 * call on each device (and the first after a cudaDeviceReset) before any stream capture.
 * Every call shares the array and it keeps the last call's contents (nothing in it needs to
 * start at zero); calls that overlap on the GPU, e.g. on two streams, race on it and must be
 * serialised by the caller.  Arguments, results and errors are otherwise exactly those of
 * ps_decode_attn. */
int ps_decode_attn_noalloc(const ps_params* params, const ps_kv_cache* cache, const void* q,
                           const int64_t* pos, void* out, float* lse, int32_t* dev_status,
                           ps_stream_t stream);

/* Bytes of device workspace ps_decode_attn_shared_prefix needs for this batch and group
 * size (the split-K partials of the window pass plus fp32 prefix partials per (sequence,
 * query head) and prefix key range).  0 on invalid arguments. */
size_t ps_decode_shared_prefix_workspace_bytes(const ps_params* params, int64_t batch,
                                               int64_t group_size);

/* Decode step for groups of sequences that share one prompt prefix.  Source: eq. A(i)
 * (§核心机制: every sequence pins its prompt as the prefix), §Kernel 实现 (the sampling code
 * sends one prompt per request; the accuracy tables average many samples of one problem):
 * the sequences of a group attend the same l_prefix rows, so those rows are read once per
 * group instead of once per sequence.  Results equal ps_decode_attn on a cache whose
 * prefix of every sequence is its group's prefix.
 *   cache->k_prefix, v_prefix : device bf16 [batch / group_size, Hkv, l_prefix, D]: the
 *                  prefix of group j is shared by sequences [j * group_size, (j+1) * group_size).
 *                  Fill it with ps_kv_append_rope on a linear cache of batch / group_size
 *                  sequences (ring NULL, positions 0 .. l_prefix - 1).
 *   cache->k_ring, v_ring     : device bf16 [batch, Hkv, W, D], one ring per sequence; append
 *                  decode tokens with a ring-only cache (prefix pointers NULL).
 *   cache->batch  : number of sequences, a multiple of group_size.
 *   group_size    : sequences per shared prefix, >= 1.
 *   q, pos, out, lse, dev_status : as ps_decode_attn.
 *   workspace, ws_bytes : device scratch of at least
 *                  ps_decode_shared_prefix_workspace_bytes(), 256-byte aligned.
 * The prefix pass runs on an internal side stream of the library (one per device, created
 * on first use), forked from `stream` before the window decode and joined before the final
 * merge, so it overlaps the window decode; the call stays asynchronous and ordered on
 * `stream`.
 * Requires l_prefix >= 1, 1 <= Hq / Hkv <= 8 and batch <= 1024 (PS_ERR_UNSUPPORTED). */
int ps_decode_attn_shared_prefix(const ps_params* params, const ps_kv_cache* cache,
                                 int64_t group_size, const void* q, const int64_t* pos,
                                 void* out, float* lse, void* workspace, size_t ws_bytes,
                                 int32_t* dev_status, ps_stream_t stream);

/* Append tokens to the pinned prefix at run time.  Source: §局限 of "Prefix Sliding 完全拆解"
 * (a mechanism for the model to append important tokens to the prefix; whether later user
 * messages of a conversation should be pinned into the prefix).  A promoted token is
 * never evicted: from then on every query sees it, together with eq. A(i)'s set.
 * The prefix store has room for appended tokens: cache->k_prefix / v_prefix are
 * [batch, Hkv, prefix_capacity, D]; rows [0, l_prefix) hold the prompt (fill them with
 * ps_kv_append_rope on a linear view of the store, ring NULL, params with
 * l_prefix = prefix_capacity), rows [l_prefix, l_prefix + pin_count[b]) the promoted
 * tokens in ascending position order.  Decode-phase appends go through a ring-only view
 * (prefix pointers NULL).
 *   pin_count : device int32 [batch], promoted tokens so far (start at 0); updated.
 *   pin_pos   : device int64 [batch, prefix_capacity - l_prefix], their positions; updated.
 *   t0, t1    : device int64 [batch]; tokens [t0[b], t1[b]) of sequence b are promoted
 *               (t1 <= t0: nothing).  They must still be in the window of pos[b] (the latest
 *               appended position): l_prefix <= t0, t0 > pos - W, t1 - 1 <= pos; follow the
 *               previous promoted position; and fit the capacity.  Otherwise the sequence
 *               is left unchanged and PS_DEV_POS_RANGE is set.
 * Their K/V rows are copied from the ring unchanged (Continue PE: already rotated). */
int ps_kv_pin(const ps_params* params, const ps_kv_cache* cache, int32_t prefix_capacity,
              int32_t* pin_count, int64_t* pin_pos, const int64_t* t0, const int64_t* t1,
              const int64_t* pos, int32_t* dev_status, ps_stream_t stream);

/* Bytes of device workspace ps_decode_attn_pinned needs.  0 on invalid arguments. */
size_t ps_decode_pinned_workspace_bytes(const ps_params* params, int64_t batch,
                                        int32_t prefix_capacity);

/* Decode step with promoted tokens (ps_kv_pin): the query at pos[b] attends the prompt
 * rows, every promoted token at a position <= pos[b], and the window, each key once (a
 * promoted token still inside the window is read from the ring).  Promoted rows whose
 * positions precede the window start are read with the prefix (a binary search over
 * pin_pos per sequence).  Other arguments and results as ps_decode_attn. */
int ps_decode_attn_pinned(const ps_params* params, const ps_kv_cache* cache,
                          int32_t prefix_capacity, const int32_t* pin_count,
                          const int64_t* pin_pos, const void* q, const int64_t* pos, void* out,
                          float* lse, void* workspace, size_t ws_bytes, int32_t* dev_status,
                          ps_stream_t stream);

/* Paged store ("Prefix Sliding 完全拆解", §核心机制: with paged block management every
 * sequence can pre-allocate a fixed number of blocks, since it never holds more than
 * L_prefix + W tokens).  K and V of all sequences live in one pool of 64-token blocks:
 *   k_pool, v_pool : device bf16 [n_blocks, Hkv, 64, D].
 *   block_table    : device int32 [batch, table_stride]; for sequence b, entries
 *                    0 .. ceil(L_prefix / 64) - 1 are its prefix blocks (position p < L_prefix
 *                    is row p % 64 of entry p / 64) and the next W / 64 entries its ring blocks
 *                    (ring slot s = (p - L_prefix) mod W is row s % 64 of entry
 *                    ceil(L_prefix / 64) + s / 64).  Sequences may share blocks, e.g. the
 *                    prefix blocks of one prompt.
 * Rows of a block that no visible position maps to (the tail of the last prefix block, ring
 * rows not yet written) may hold anything, NaN included: they never reach the result.
 * Requires W a multiple of 64 and table_stride >= ceil(L_prefix / 64) + W / 64.  A table
 * entry outside [0, n_blocks) sets PS_DEV_POS_RANGE: the append writes nothing for that
 * token and the decode reads zeros for that block. */
int ps_kv_append_rope_paged(const ps_params* params, void* k_pool, void* v_pool,
                            int64_t n_blocks, const int32_t* block_table, int32_t table_stride,
                            int64_t batch, const void* k_new, const void* v_new, void* q_inout,
                            const int64_t* pos0, int32_t T, int32_t* dev_status,
                            ps_stream_t stream);

/* Decode step over a paged store: results equal ps_decode_attn on the same keys; every
 * 64-row tile is one block, loaded where the table points.  Other arguments, the workspace
 * (ps_decode_workspace_bytes) and errors as ps_decode_attn. */
int ps_decode_attn_paged(const ps_params* params, void* k_pool, void* v_pool, int64_t n_blocks,
                         const int32_t* block_table, int32_t table_stride, int64_t batch,
                         const void* q, const int64_t* pos, void* out, float* lse,
                         void* workspace, size_t ws_bytes, int32_t* dev_status,
                         ps_stream_t stream);

/* Bytes of device workspace ps_full_attn_ref needs (same split-K layout as decode). */
size_t ps_full_attn_workspace_bytes(const ps_params* params, int64_t batch, int64_t lmax);

/* Full causal attention comparator (the baseline the pages compare against, §Kernel 实现
 * and Table 1 full-attention row): the query at pos[b] attends every key in [0, pos[b]].
 *   k_full, v_full : device bf16 [batch, Hkv, lmax, D], keys already rotated (fill it with
 *                    ps_kv_append_rope on a cache with l_prefix = lmax, ring NULL).
 *   pos[b] >= lmax sets PS_DEV_POS_RANGE and skips sequence b.
 * params->l_prefix and params->window are ignored. Other arguments as ps_decode_attn. */
int ps_full_attn_ref(const ps_params* params, const void* k_full, const void* v_full,
                     int64_t lmax, const void* q, const int64_t* pos, int64_t batch, void* out,
                     float* lse, void* workspace, size_t ws_bytes, int32_t* dev_status,
                     ps_stream_t stream);

/* Prefill tile geometry (query rows Bq, key rows Bk) the masked prefill kernel uses. */
int ps_prefill_tile_geometry(int32_t* bq, int32_t* bk);

/* Number of non-SKIP tiles of the prefill plan for one (batch, head), host-computed from
 * the same closed forms the device planner uses.  Returns < 0 on invalid arguments. */
int64_t ps_prefill_plan_tiles(const ps_params* params, int64_t seq);

/* Bytes of device workspace ps_masked_prefill_attn needs. */
size_t ps_prefill_workspace_bytes(const ps_params* params, int64_t batch, int64_t seq);

/* Masked prefill / truncated-backprop context forward over sequence indices [0, seq).
 * Source: eq. A(i) (§核心机制); §Kernel 实现 (two-level filtering); §截断回传 (the trainer
 * runs the forward over the last 4W tokens of a rollout).
 * Row i attends V(i) with positions taken as sequence indices: the first l_prefix
 * indices are the prefix.  With window >= seq this is dense causal attention.
 *   q      : device bf16 [batch, seq, Hq, D], already rotated.
 *   k, v   : device bf16 [batch, seq, Hkv, D], k already rotated.
 *   out    : device bf16 [batch, seq, Hq, D].
 *   lse    : device fp32 [batch, Hq, seq] or NULL (natural log).
 *   tile_plan : device int32 [tile_plan_cap, 3] or NULL.  When given, receives the plan
 *           the kernel ran: rows (q_tile, k_tile, flag), q-tile-major, ascending k_tile,
 *           SKIP tiles omitted (flag PS_TILE_FULL or PS_TILE_PARTIAL).
 *   n_tiles : host int64 or NULL; receives the number of plan rows.
 *   workspace, ws_bytes : device scratch of at least ps_prefill_workspace_bytes() (it holds
 *           the tile plan the kernel walks).
 *   dev_status : device int32 or NULL (PS_DEV_TIMEOUT only).
 * Requires seq >= 1 and Hq / Hkv integral.  tile_plan_cap smaller than the plan is
 * PS_ERR_INVALID_ARG. */
int ps_masked_prefill_attn(const ps_params* params, const void* q, const void* k, const void* v,
                           int64_t batch, int64_t seq, void* out, float* lse, int32_t* tile_plan,
                           int64_t tile_plan_cap, int64_t* n_tiles, void* workspace,
                           size_t ws_bytes, int32_t* dev_status, ps_stream_t stream);

/* Bytes of device workspace recommended for ps_masked_prefill_attn_bwd over `batch`
 * sequences: the tile plan, a work counter, and per sequence of one pass two fp32 row
 * statistics per (head, row) padded to whole 128-row tiles and the bf16 dS^T tile of every
 * planned (query tile, key tile) pair per head (32 KB each).  The batch runs in passes: one
 * pass when that store stays within 4 GiB, else passes of as many sequences as fit in 4 GiB
 * (so the size stops growing with the batch).  The value for batch = 1 is the minimum the
 * call accepts; a workspace between the two runs passes of as many sequences as it holds. */
size_t ps_prefill_bwd_workspace_bytes(const ps_params* params, int64_t batch, int64_t seq);

/* Backward of ps_masked_prefill_attn: gradients of the masked attention with respect to
 * q, k and v.  Source: §截断回传 of "Prefix Sliding 完全拆解" (the trainer back-propagates
 * through the masked attention over the last 4W tokens of a rollout), eq. A(i) for the
 * mask, §Kernel 实现 for the tile skipping (the same plan as the forward).
 * With P the masked softmax of the forward and D_i = <dout_i, out_i>:
 *   dv_j = sum_i P_ij dout_i,  dS_ij = P_ij (<dout_i, v_j> - D_i),
 *   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,
 * dk and dv summed over the query heads that share a KV head.
 *   q, k, v  : the forward's inputs (layouts as ps_masked_prefill_attn).
 *   out      : device bf16 [batch, seq, Hq, D], the forward's output.
 *   dout     : device bf16 [batch, seq, Hq, D], gradient of the loss with respect to out.
 *   lse      : device fp32 [batch, Hq, seq], the forward's log-sum-exp (required).
 *   dq       : device bf16 [batch, seq, Hq, D] (written).
 *   dk, dv   : device bf16 [batch, seq, Hkv, D] (written).
 *   workspace, ws_bytes : device scratch of at least ps_prefill_bwd_workspace_bytes() for
 *              batch 1, 256-byte aligned; results do not depend on its size (every pass
 *              covers whole sequences).  Smaller: PS_ERR_WORKSPACE.
 *   dev_status : device int32 or NULL (PS_DEV_TIMEOUT only).
 * Requires seq >= 1, Hq / Hkv integral.  All of q, k, v, out, dout, dq, dk, dv 16-byte
 * aligned.  Outputs are written in full (no accumulation into existing values). */
int ps_masked_prefill_attn_bwd(const ps_params* params, const void* q, const void* k,
                               const void* v, const void* out, const void* dout,
                               const float* lse, int64_t batch, int64_t seq, void* dq, void* dk,
                               void* dv, void* workspace, size_t ws_bytes, int32_t* dev_status,
                               ps_stream_t stream);

/* Introspection for bit-exact checks: the visible-range descriptor the decode kernel
 * uses, computed by the same device code.  ranges_out: device int32 [batch, 4] =
 * (pre_len, seg0_start, seg0_len, seg1_len): the prefix rows [0, pre_len) and the ring
 * slots [seg0_start, seg0_start + seg0_len) then [0, seg1_len).  An empty window reports
 * (.., 0, 0, 0).  A position < 0 reports (0, 0, 0, 0). */
int ps_decode_visible_ranges(const ps_params* params, const int64_t* pos, int64_t batch,
                             int32_t* ranges_out, ps_stream_t stream);

/* Diagnostic of the bounded waits every kernel uses (the pages have no counterpart): one
 * CTA waits, with the library's own wait, on a shared-memory barrier phase that nothing
 * completes.  After the wait limit (about one second) the wait gives up, the kernel ORs
 * PS_DEV_TIMEOUT into *dev_status and returns, so the stream moves on and the context stays
 * usable.  Lets a test check on the device that a stalled wait ends with a status, not a
 * hang.
 *   dev_status : device int32, 4-byte aligned (required).
 * Asynchronous on `stream`; about one second of device time. */
int ps_check_wait_timeout(int32_t* dev_status, ps_stream_t stream);

/* Thread-local description of the last host-side failure of this thread ("" if none). */
const char* ps_last_error(void);

/* Library version string. */
const char* ps_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PS_H_ */
