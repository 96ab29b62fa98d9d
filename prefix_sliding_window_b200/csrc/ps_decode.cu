// Split-K decode attention for the Prefix Sliding KV store (and the full-attention
// comparator over a linear cache), sm_100a.
//
// What it computes ("Prefix Sliding 完全拆解", §核心机制, eq. A(i)): the query of sequence b
// at position p attends only its visible keys, the prefix rows [0, min(p+1, Lp)) and the
// window positions [max(Lp, p+1-W), p+1), which live in ring slots (pos - Lp) mod W.  Only
// those rows are read ("§Kernel 实现": evicted keys are never loaded), so the bytes read per
// step stop growing once the window is full (eq. L_total).
//
// Work units are (sequence, KV head) pairs; a unit's visible keys are cut into 64-row TMA
// tiles (make_tiling).  Two schedules:
//  * per-unit: when there are at least as many units as CTA slots (148 SMs x 2), one CTA
//    per unit, written straight to `out`;
//  * stream-K: otherwise one wave of CTAs (up to 2 per SM; a multiple of the unit count when
//    that fills at least 5/6 of the slots) takes equal contiguous shares of the global tile
//    sequence (all units' tiles back to back), so every SM streams the same number of bytes
//    whatever the positions are.  A CTA whose share crosses a unit boundary flushes a partial
//    (o, lse) per unit piece; merge_kernel combines the pieces.
// Inside a CTA:
//  * warp 4 is the producer: one lane issues four 3-D TMA loads per tile (K and V, two
//    64-column halves each, 128-byte swizzle) into a 3-stage mbarrier ring;
//  * warps 0-3 consume 16 keys each per tile with warp-level bf16 tensor-core MMAs in fp32:
//      S^T[16 keys x 8 heads] = K[16 x 128] . Q^T       (GQA: the 8 query heads of the
//                                                          KV head share every K/V load)
//      O^T[128 x 8 heads]    += V^T[128 x 16] . P^T
//    P^T goes from the accumulator layout to the operand layout with movmatrix; softmax is
//    online, in base 2, with warp-shuffle max reductions;
//  * the four warps' (m, l, O) states are merged through shared memory.
#include <cuda_bf16.h>
#include <math.h>

#include "ps_device.cuh"
#include "ps_internal.h"
#include "ps_ranges.cuh"

#include <mutex>
#include <string>

namespace ps {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kBoxBytes = kDecodeTile * 128;  // 64 rows x 64 bf16
constexpr int kTileBytes = 2 * kBoxBytes;     // one K (or V) tile: two column halves
constexpr int kStageBytes = 2 * kTileBytes;   // K + V
constexpr int kStages = 3;
constexpr int kCtasPerSm = 2;
constexpr int kMaxStreamKSeqs = 1024;  // stream-K runs only when units < CTA slots
// Small batches get one CTA per this many tiles (up to the CTA slots): each CTA's first TMA
// round trip is the latency floor, and every further CTA adds a piece to merge.  At batch 1,
// 612 visible keys (24 tiles), 2 gave 8.6 us per graph-launched step against 9.1 us with 4 and
// 10.3 us with 1.
constexpr int kMinTilesPerCta = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// decode_kernel modes (a template parameter: each mode's extra registers stay out of the
// others)
constexpr int kPlain = 0;  // ps_decode_attn and its variants
constexpr int kReset = 1;  // Reset PE: prefix tiles see the query at its Reset-PE id

// shared memory: stages | barriers (2 x STAGES) | flush area [2][32 lanes][36] | prefix
constexpr size_t kFlushFloats = 2 * 32 * 36;
constexpr size_t smem_bytes(int stages) {
  return 1024 + size_t(stages) * kStageBytes + 64 + kFlushFloats * 4 +
         (kMaxStreamKSeqs + 1) * 4;
}

struct DecodeArgs {
  const __nv_bfloat16* q;
  const int64_t* pos;
  __nv_bfloat16* out;
  float* lse;
  float* ws_o;      // stream-K: [slots, 8, D] normalised partial outputs
  float* ws_lse;    // stream-K: [slots, 8] base-2 lse of each partial
  int32_t* status;
  int32_t batch, hq, hkv, group;
  int32_t lp, w, dim0;
  int32_t streamk, full_mode;
  int64_t lmax;
  float scale_log2;
  int32_t skip_prefix;     // shared-prefix decode: window rows only
  // Reset PE: prefix tiles use the query rotated by delta = L_prefix + |window| - 1 - p
  // more (its Reset-PE id); inv_freq = theta^(-2i/D) in float64
  int32_t reset_pe;
  // launched right after a one-token append at pos (ps_decode_step): only the tile holding
  // each sequence's newest row and the rotated q depend on that kernel, so everything else
  // may stream before the programmatic wait
  int32_t after_append;
  // paged store: K/V of every (sequence, KV head) in 64-row blocks of one pool
  // [n_blocks][Hkv][64][D]; logical block i of sequence b is table[b * table_stride + i]
  // (prefix blocks first, then W / 64 ring blocks)
  int32_t paged;
  const int32_t* table;
  int32_t table_stride, pre_blocks;
  int64_t n_blocks;
  double inv_freq[kHeadDim / 2];
  // tokens appended to the pinned prefix: rows [L_prefix, L_prefix + pin_count[b]) of the
  // prefix store hold the promoted positions pin_pos[b][0..) (ascending)
  const int32_t* pin_count;
  const int64_t* pin_pos;
  int32_t pin_cap;
};

// Offset of the 16-byte chunk `chunk` (0..7) of box row `row` under the 128-byte swizzle
// TMA applies (chunk index XOR row mod 8; boxes start 1024-byte aligned).
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return uint32_t(row) * 128u + (uint32_t(chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ bool bad_position(const DecodeArgs& a, int64_t p) {
  return (p < 0) || (a.full_mode && p >= a.lmax);
}

__device__ __forceinline__ DecodeTiling tiling_of(const DecodeArgs& a, int64_t b, int64_t p) {
  VisibleRanges r{0, 0, 0, 0};
  if (!bad_position(a, p)) {
    if (a.full_mode)
      r.pre_len = static_cast<int32_t>(p + 1);
    else
      r = visible_ranges(p, a.lp, a.w);
    if (a.skip_prefix) r.pre_len = 0;  // the shared-prefix pass covers those rows
    if (a.pin_count && p >= a.lp) {
      // promoted rows whose positions precede the window start are read with the prefix;
      // the rest are still in the window (ascending positions: a binary search)
      int64_t ws = p + 1 - a.w;
      if (ws < a.lp) ws = a.lp;
      const int64_t* pp = a.pin_pos + b * a.pin_cap;
      int lo = 0, hi = a.pin_count[b];
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (pp[mid] < ws) lo = mid + 1; else hi = mid;
      }
      r.pre_len += lo;
    }
  }
  return a.paged ? make_tiling_paged(r) : make_tiling(r, a.dim0, a.w);
}

// Walks a contiguous range of the global tile sequence: unit u = b * hkv + h owns tiles
// [hkv * pref[b] + h * cnt_b, ... + cnt_b), cnt_b = pref[b+1] - pref[b].
struct TileWalker {
  int64_t t, t_end;      // global tile cursor and end
  int64_t pu, pu1;       // tile range of the current unit
  int32_t b, h;          // current unit
  DecodeTiling tiling;   // tiling of sequence b

  __device__ void enter_unit(const DecodeArgs& a, const int32_t* pref) {
    const int64_t cnt = pref[b + 1] - pref[b];
    pu = (int64_t)a.hkv * pref[b] + h * cnt;
    pu1 = pu + cnt;
    tiling = tiling_of(a, b, a.pos[b]);
  }
  // position the walker on global tile t0 (t0 < total)
  __device__ void seek(const DecodeArgs& a, const int32_t* pref, int64_t t0) {
    int lo = 0, hi = a.batch - 1;  // largest b with hkv * pref[b] <= t0
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((int64_t)a.hkv * pref[mid] <= t0) lo = mid; else hi = mid - 1;
    }
    b = lo;
    const int64_t cnt = pref[b + 1] - pref[b];
    const int64_t off = t0 - (int64_t)a.hkv * pref[b];  // < hkv * cnt
    h = static_cast<int32_t>(off < (int64_t(1) << 32) ? uint32_t(off) / uint32_t(cnt)
                                                       : off / cnt);
    t = t0;
    enter_unit(a, pref);
  }
  // move to the next unit that owns tiles, without its tiling (for a look-ahead)
  __device__ void next_unit_light(const DecodeArgs& a, const int32_t* pref) {
    do {
      if (++h == a.hkv) {
        h = 0;
        ++b;
      }
    } while (pref[b + 1] == pref[b]);
  }
  // move to the next unit that owns tiles
  __device__ void next_unit(const DecodeArgs& a, const int32_t* pref) {
    do {
      if (++h == a.hkv) {
        h = 0;
        ++b;
      }
    } while (pref[b + 1] == pref[b]);
    enter_unit(a, pref);
  }
};

// Merges another (m, l, O) state into the registers of this lane (same fragment layout).
__device__ __forceinline__ void merge_state(float& m0, float& m1, float& l0, float& l1,
                                            float (&o)[8][4], const float* other) {
  const float om0 = other[32], om1 = other[33], ol0 = other[34], ol1 = other[35];
  const float M0 = fmaxf(m0, om0), M1 = fmaxf(m1, om1);
  const float fa0 = (m0 == -INFINITY) ? 0.f : fast_exp2(m0 - M0);
  const float fb0 = (om0 == -INFINITY) ? 0.f : fast_exp2(om0 - M0);
  const float fa1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - M1);
  const float fb1 = (om1 == -INFINITY) ? 0.f : fast_exp2(om1 - M1);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    o[j][0] = fa0 * o[j][0] + fb0 * other[4 * j + 0];
    o[j][1] = fa1 * o[j][1] + fb1 * other[4 * j + 1];
    o[j][2] = fa0 * o[j][2] + fb0 * other[4 * j + 2];
    o[j][3] = fa1 * o[j][3] + fb1 * other[4 * j + 3];
  }
  l0 = fa0 * l0 + fb0 * ol0;
  l1 = fa1 * l1 + fb1 * ol1;
  m0 = M0;
  m1 = M1;
}

__device__ __forceinline__ void store_state(float* dst, float m0, float m1, float l0, float l1,
                                            const float (&o)[8][4]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    dst[4 * j + 0] = o[j][0];
    dst[4 * j + 1] = o[j][1];
    dst[4 * j + 2] = o[j][2];
    dst[4 * j + 3] = o[j][3];
  }
  dst[32] = m0;
  dst[33] = m1;
  dst[34] = l0;
  dst[35] = l1;
}

// MODE: kPlain or kReset (prefix tiles see the query at its renumbered id).  A template
// parameter, not a run-time flag, so the plain decode carries none of Reset PE's registers.
// Two CTAs of 5 warps per SM need at most 168 registers per thread (10 warps on 4 SMSPs: 3
// warps x 168 x 32 fit one SMSP's 16K registers); the bound keeps both modes there, and the
// stream-K grid is sized for two per SM.
template <int STAGES, int MODE>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    decode_kernel(const __grid_constant__ CUtensorMap mk0, const __grid_constant__ CUtensorMap mv0,
                  const __grid_constant__ CUtensorMap mk1, const __grid_constant__ CUtensorMap mv1,
                  const DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * kStageBytes);
  uint64_t* empty = full + STAGES;
  float* flush = reinterpret_cast<float*>(smem + STAGES * kStageBytes + 64);  // [2][32][36]
  int32_t* pref = reinterpret_cast<int32_t*>(flush + kFlushFloats);            // [batch + 1]
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  if (warp == kConsumerWarps && lane == 0) {
    prefetch_tensormap(&mk0);
    prefetch_tensormap(&mv0);
    prefetch_tensormap(&mk1);
    prefetch_tensormap(&mv1);
  }
  // launched with programmatic serialization: everything above overlapped the previous
  // kernel (usually the append); positions, q and the cache are read only after this
  if (!a.after_append) pdl_wait();
  pdl_trigger();  // the merge may be scheduled now; it waits for this grid to finish

  // ---------------------------------------------------------------- work range
  TileWalker wk;
  if (a.streamk) {
    // tiles per sequence, then an inclusive scan (batch <= kMaxStreamKSeqs)
    for (int b = threadIdx.x; b < a.batch; b += kThreads) {
      const int64_t p = a.pos[b];
      const int32_t cnt = tiling_of(a, b, p).total;
      pref[b + 1] = cnt;
      if (blockIdx.x == 0 && cnt == 0 && bad_position(a, p) && a.status)
        atomicOr(a.status, p < 0 ? PS_DEV_BAD_POS : PS_DEV_POS_RANGE);
    }
    if (threadIdx.x == 0) pref[0] = 0;
    __syncthreads();
    if (warp == 0) {
      int32_t carry = 0;
      for (int base = 1; base <= a.batch; base += 32) {
        const int i = base + lane;
        int32_t v = i <= a.batch ? pref[i] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int32_t u = __shfl_up_sync(0xffffffffu, v, off);
          if (lane >= off) v += u;
        }
        if (i <= a.batch) pref[i] = v + carry;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
    }
    __syncthreads();
    const int64_t total = (int64_t)a.hkv * pref[a.batch];
    // this CTA's share [total c / G, total (c + 1) / G), in 32 bits when total G fits
    int64_t t0, t1;
    if (total * gridDim.x < (int64_t(1) << 32)) {
      const uint32_t tt = static_cast<uint32_t>(total);
      t0 = (tt * blockIdx.x) / gridDim.x;
      t1 = (tt * (blockIdx.x + 1)) / gridDim.x;
    } else {
      t0 = total * blockIdx.x / gridDim.x;
      t1 = total * (blockIdx.x + 1) / gridDim.x;
    }
    wk.t_end = t1;
    if (t0 < t1) {
      wk.seek(a, pref, t0);
    } else {
      wk.t = t0;
    }
  } else {
    __syncthreads();
    const int unit = blockIdx.x;
    wk.b = unit / a.hkv;
    wk.h = unit % a.hkv;
    const int64_t p = a.pos[wk.b];
    if (bad_position(a, p) && threadIdx.x == 0 && wk.h == 0 && a.status)
      atomicOr(a.status, p < 0 ? PS_DEV_BAD_POS : PS_DEV_POS_RANGE);
    wk.tiling = tiling_of(a, wk.b, p);
    wk.t = 0;
    wk.t_end = wk.tiling.total;
    wk.pu = 0;
    wk.pu1 = wk.t_end;
  }
  const int ntiles = static_cast<int>(wk.t_end - wk.t);

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && ntiles > 0) {
      const uint64_t pol = l2_policy_evict_first();
      int issued = 0;
      bool waited = !a.after_append;
      TileWalker pw = wk;
      for (int i = 0; i < ntiles; ++i, ++pw.t) {
        if (pw.t >= pw.pu1) pw.next_unit(a, pref);
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (i >= STAGES && !mbar_wait(&empty[s], ph ^ 1, a.status)) break;
        const DecodeTile d = tiling_tile(pw.tiling, static_cast<int32_t>(pw.t - pw.pu));
        if (!waited) {
          // the newest row of sequence b: prefix row p, or ring slot (p - Lp) mod W
          const int64_t p = a.pos[pw.b];
          const bool pre = a.full_mode || p < a.lp;
          const int64_t row = pre ? p : mod_nonneg(p - a.lp, a.w);
          if (d.map_id == (pre ? 0 : 1) && row >= d.row0 + d.lo && row < d.row0 + d.hi) {
            pdl_wait();
            waited = true;
          }
        }
        const CUtensorMap* mk = d.map_id ? &mk1 : &mk0;
        const CUtensorMap* mv = d.map_id ? &mv1 : &mv0;
        const int unit = pw.b * a.hkv + pw.h;
        uint8_t* st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        if (a.paged) {
          // one tile = one block of the pool (a block id out of range reads zeros: TMA
          // clips coordinates to the pool; it is flagged)
          const int32_t blk =
              a.table[(int64_t)pw.b * a.table_stride + (d.map_id ? a.pre_blocks : 0) +
                      d.row0 / kDecodeTile];
          if ((blk < 0 || blk >= a.n_blocks) && a.status) atomicOr(a.status, PS_DEV_POS_RANGE);
          tma_load_4d(st, &mk0, 0, 0, pw.h, blk, &full[s]);
          tma_load_4d(st + kBoxBytes, &mk0, 64, 0, pw.h, blk, &full[s]);
          tma_load_4d(st + kTileBytes, &mv0, 0, 0, pw.h, blk, &full[s]);
          tma_load_4d(st + kTileBytes + kBoxBytes, &mv0, 64, 0, pw.h, blk, &full[s]);
        } else {
          tma_load_3d_hint(st, mk, 0, d.row0, unit, &full[s], pol);
          tma_load_3d_hint(st + kBoxBytes, mk, 64, d.row0, unit, &full[s], pol);
          tma_load_3d_hint(st + kTileBytes, mv, 0, d.row0, unit, &full[s], pol);
          tma_load_3d_hint(st + kTileBytes + kBoxBytes, mv, 64, d.row0, unit, &full[s], pol);
        }
        issued = i + 1;
      }
      // every issued copy must land before the CTA may exit or reuse shared memory
      for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1, a.status);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int qh = lane >> 2;  // query head within the group (MMA column)
    const int qq = lane & 3;
    const float sl2 = a.scale_log2;
    const int arow = 16 * warp + (lane & 15);  // ldmatrix row for K
    const int achunk = lane >> 4;              // 0/1: k 0-7 or 8-15
    const int vkey = 16 * warp + (lane & 7) + ((lane >> 4) << 3);
    const int vdoff = ((lane >> 3) & 1) << 3;
    const int r0 = 16 * warp + (lane >> 2);
    const int r1 = r0 + 8;

    float o[8][4];
    float m0, m1, l0, l1;
    uint32_t qf[8][2];
    uint32_t qp[8][2];  // Reset PE: the query at its Reset-PE id, for prefix tiles
    // dst = R_shift src on this lane's fragments (rotate-half RoPE composes: R_a R_b =
    // R_(a+b)).  This lane's pairs are (d, d + 64) for d = 16 ks + 8 r + 2 qq + {0, 1},
    // ks < 4: fragments ks and ks + 4.  The lane forms the angles of frequencies d = lane and
    // lane + 32 (rope_cos_sin: float64, reduced modulo 2 pi, as in the append); every lane
    // then reads the 16 it needs with shuffles (each is needed by the 8 lanes of one qq).
    // src and dst may be the same array.
    auto rope_frag = [&](const uint32_t (&src)[8][2], int64_t shift, uint32_t (&dst)[8][2]) {
      float cw[2], sw[2];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float2 cs = rope_cos_sin(double(shift), a.inv_freq[lane + 32 * hf]);
        cw[hf] = cs.x;
        sw[hf] = cs.y;
      }
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const uint32_t lo = src[ks][r], hi = src[ks + 4][r];
          const float2 x1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lo));
          const float2 x2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi));
          float c[2], sn[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int d = 16 * ks + 8 * r + 2 * qq + e;  // d >> 5 == ks >> 1
            c[e] = __shfl_sync(0xffffffffu, cw[ks >> 1], d & 31);
            sn[e] = __shfl_sync(0xffffffffu, sw[ks >> 1], d & 31);
          }
          dst[ks][r] = pack_bf16x2(rope_lo(x1.x, x2.x, c[0], sn[0]), rope_lo(x1.y, x2.y, c[1], sn[1]));
          dst[ks + 4][r] =
              pack_bf16x2(rope_hi(x1.x, x2.x, c[0], sn[0]), rope_hi(x1.y, x2.y, c[1], sn[1]));
        }
      }
    };
    // Reset PE: prefix tiles see the query at its Reset-PE id L_prefix + |window| - 1, i.e.
    // rotated by delta = L_prefix - max(L_prefix, p + 1 - W) <= 0 more (0 while nothing is
    // evicted)
    auto rotate_prefix_q = [&](int64_t p) {
      int64_t ws = p + 1 - a.w;
      if (ws < a.lp) ws = a.lp;
      rope_frag(qf, (int64_t)a.lp - ws, qp);
    };
    auto reset = [&]() {
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    };
    auto load_q = [&](int b, int h) {
      if (qh < a.group) {
        const __nv_bfloat16* qrow = a.q + ((int64_t)b * a.hq + h * a.group + qh) * kHeadDim;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          qf[ks][0] = *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * qq);
          qf[ks][1] = *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * qq);
        }
      } else {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) qf[ks][0] = qf[ks][1] = 0u;
      }
    };
    // Folds the four warps' states of the current unit into warp 0 (two rounds through
    // shared memory) and writes the result: to `out` for a whole unit, to the workspace
    // for a stream-K piece.
    auto flush_unit = [&](int b, int h) {
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
      }
      if (warp >= 2) store_state(flush + ((warp - 2) * 32 + lane) * 36, m0, m1, l0, l1, o);
      named_bar_sync(1, kConsumerThreads);
      if (warp < 2) merge_state(m0, m1, l0, l1, o, flush + (warp * 32 + lane) * 36);
      named_bar_sync(1, kConsumerThreads);
      if (warp == 1) store_state(flush + lane * 36, m0, m1, l0, l1, o);
      named_bar_sync(1, kConsumerThreads);
      if (warp == 0) {
        merge_state(m0, m1, l0, l1, o, flush + lane * 36);
        const int unit = b * a.hkv + h;
        const int64_t slot = (int64_t)unit + blockIdx.x;  // unique per (unit, CTA) piece
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int hh = 2 * qq + e;
          const float m = e ? m1 : m0;
          const float l = e ? l1 : l0;
          const float inv = l > 0.f ? 1.f / l : 0.f;
          const float lse2 = l > 0.f ? m + log2f(l) : -INFINITY;
          if (hh < a.group) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int d0 = 16 * j + (lane >> 2);
              const float v0 = o[j][e] * inv, v1 = o[j][2 + e] * inv;
              if (a.streamk) {
                float* dst = a.ws_o + (slot * 8 + hh) * kHeadDim;
                dst[d0] = v0;
                dst[d0 + 8] = v1;
              } else {
                __nv_bfloat16* dst = a.out + ((int64_t)b * a.hq + h * a.group + hh) * kHeadDim;
                dst[d0] = __float2bfloat16_rn(v0);
                dst[d0 + 8] = __float2bfloat16_rn(v1);
              }
            }
            if (lane < 4) {
              if (a.streamk)
                a.ws_lse[slot * 8 + hh] = lse2;
              else if (a.lse)
                a.lse[(int64_t)b * a.hq + h * a.group + hh] = lse2 * kLn2;
            }
          }
        }
      }
      named_bar_sync(1, kConsumerThreads);  // the flush area is free again
    };

    reset();
    TileWalker cw = wk;
    uint32_t qn[8][2];  // q of the next unit, prefetched
    auto prefetch_next_q = [&](const TileWalker& w) {
      if (w.pu1 < w.t_end) {
        TileWalker nx = w;
        nx.next_unit_light(a, pref);
        if (qh < a.group) {
          const __nv_bfloat16* qrow =
              a.q + ((int64_t)nx.b * a.hq + nx.h * a.group + qh) * kHeadDim;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            qn[ks][0] = *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * qq);
            qn[ks][1] = *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * qq);
          }
        } else {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) qn[ks][0] = qn[ks][1] = 0u;
        }
      }
    };
    if (a.after_append) pdl_wait();  // q is rotated by the append just before
    if (ntiles > 0) {
      load_q(cw.b, cw.h);
      if (MODE == kReset) rotate_prefix_q(a.pos[cw.b]);
      prefetch_next_q(cw);
    }
    bool alive = true;
    for (int i = 0; i < ntiles; ++i, ++cw.t) {
      if (cw.t >= cw.pu1) {
        flush_unit(cw.b, cw.h);
        cw.next_unit(a, pref);
        reset();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          qf[ks][0] = qn[ks][0];
          qf[ks][1] = qn[ks][1];
        }
        if (MODE == kReset) rotate_prefix_q(a.pos[cw.b]);
        prefetch_next_q(cw);
      }
      const int s = i % STAGES;
      // warp-uniform outcome: ldmatrix / mma.sync below are warp-collective
      if (alive && !__all_sync(0xffffffffu, mbar_wait(&full[s], (i / STAGES) & 1, a.status)))
        alive = false;
      if (!alive) continue;  // keep the flush barriers in step with the other warps
      const DecodeTile d = tiling_tile(cw.tiling, static_cast<int32_t>(cw.t - cw.pu));
      const uint32_t kbase = smem_u32(smem + s * kStageBytes);
      const uint32_t vbase = kbase + kTileBytes;

      float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a0, a1, a2, a3;
        const uint32_t addr =
            kbase + (ks >> 2) * kBoxBytes + swz(arow, ((ks & 3) << 1) + achunk);
        ldmatrix_x4(addr, a0, a1, a2, a3);
        // Reset PE: prefix tiles (map 0) see the query at its Reset-PE id
        const bool pre_q = MODE == kReset && d.map_id == 0;
        mma_bf16_16816(sc, a0, a1, a2, a3, pre_q ? qp[ks][0] : qf[ks][0],
                       pre_q ? qp[ks][1] : qf[ks][1]);
      }
      const bool v0 = (r0 >= d.lo) && (r0 < d.hi);
      const bool v1 = (r1 >= d.lo) && (r1 < d.hi);
      const float x0 = v0 ? sc[0] * sl2 : -INFINITY;
      const float x1 = v0 ? sc[1] * sl2 : -INFINITY;
      const float x2 = v1 ? sc[2] * sl2 : -INFINITY;
      const float x3 = v1 ? sc[3] * sl2 : -INFINITY;
      float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float ref0 = (mn0 == -INFINITY) ? 0.f : mn0;
      const float ref1 = (mn1 == -INFINITY) ? 0.f : mn1;
      const float c0 = fast_exp2(m0 - ref0), c1 = fast_exp2(m1 - ref1);
      const float p0 = fast_exp2(x0 - ref0), p1 = fast_exp2(x1 - ref1);
      const float p2 = fast_exp2(x2 - ref0), p3 = fast_exp2(x3 - ref1);
      l0 = l0 * c0 + p0 + p2;
      l1 = l1 * c1 + p1 + p3;
      m0 = mn0;
      m1 = mn1;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        o[j][0] *= c0;
        o[j][1] *= c1;
        o[j][2] *= c0;
        o[j][3] *= c1;
      }
      const uint32_t b0 = movmatrix_trans(pack_bf16x2(p0, p1));
      const uint32_t b1 = movmatrix_trans(pack_bf16x2(p2, p3));
      // V rows outside [lo, hi) get P = 0, but 0 x NaN is NaN: a paged block's rows past
      // its segment may never have been written.  This lane's V elements are keys
      // kv, kv+1 (a0, a1) and kv+8, kv+9 (a2, a3); drop those outside the segment.
      // Full tiles take the unmasked copy of the loop (the masks fold away).
      auto pv = [&](uint32_t vm01, uint32_t vm23) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int dd = 16 * j + vdoff;
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4_trans(vbase + (dd >> 6) * kBoxBytes + swz(vkey, (dd & 63) >> 3), a0, a1,
                            a2, a3);
          mma_bf16_16816(o[j], a0 & vm01, a1 & vm01, a2 & vm23, a3 & vm23, b0, b1);
        }
      };
      if (d.lo > 0 || d.hi < kDecodeTile) {
        const int kv = 16 * warp + 2 * qq;
        auto in = [&](int k) { return k >= d.lo && k < d.hi; };
        pv((in(kv) ? 0x0000ffffu : 0u) | (in(kv + 1) ? 0xffff0000u : 0u),
           (in(kv + 8) ? 0x0000ffffu : 0u) | (in(kv + 9) ? 0xffff0000u : 0u));
      } else {
        pv(0xffffffffu, 0xffffffffu);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (ntiles > 0) {
      flush_unit(cw.b, cw.h);
    } else if (!a.streamk) {
      // a unit without visible keys (skipped position): zeros and lse = -inf
      flush_unit(wk.b, wk.h);
    }
  }
  __syncthreads();
}

// Combines the stream-K pieces of one (sequence, query head): weights 2^(lse_s - max).
// CTA c of the decode owned the global tiles [total c / grid, total (c+1) / grid) and stored
// its piece of unit u at slot u + c.  The merge recomputes that partition itself, from the
// positions (written before the decode ran), while the decode still runs: only the pieces
// are read after the programmatic wait.  One warp per (sequence, query head); lane i owns
// d = 4i .. 4i+3.
__global__ void __launch_bounds__(128)
    merge_kernel(const __grid_constant__ DecodeArgs a, int32_t grid,
                 const float* __restrict__ pre_o, const float* __restrict__ pre_lse2,
                 int32_t pre_splits) {
  __shared__ int32_t s_pref[kMaxStreamKSeqs + 1];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // tiles per sequence, exactly as the decode counts them, then an inclusive scan
  for (int i = threadIdx.x; i < a.batch; i += blockDim.x)
    s_pref[i + 1] = tiling_of(a, i, a.pos[i]).total;
  if (threadIdx.x == 0) s_pref[0] = 0;
  __syncthreads();
  if (warp == 0) {
    int32_t carry = 0;
    for (int base = 1; base <= a.batch; base += 32) {
      const int i = base + lane;
      int32_t v = i <= a.batch ? s_pref[i] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += u;
      }
      if (i <= a.batch) s_pref[i] = v + carry;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  __syncthreads();
  const int64_t bh = (int64_t)blockIdx.x * 4 + warp;
  if (bh >= (int64_t)a.batch * a.hq) return;
  const int hq = a.hq, hkv = a.hkv, group = a.group, batch = a.batch;
  const int b = static_cast<int>(bh / hq), head = static_cast<int>(bh % hq);
  const int h = head / group, hh = head % group;
  const int64_t unit = (int64_t)b * hkv + h;
  const int64_t total = (int64_t)hkv * s_pref[batch];
  const int64_t cnt = s_pref[b + 1] - s_pref[b];
  // the CTAs holding the unit's first and last tiles: the CTA owning tile t is
  // ((t + 1) grid - 1) / total
  int c_lo = 1, c_hi = 0;
  if (cnt > 0) {
    const int64_t pu = (int64_t)hkv * s_pref[b] + h * cnt;
    c_lo = static_cast<int>(((pu + 1) * grid - 1) / total);
    c_hi = static_cast<int>(((pu + cnt) * grid - 1) / total);
  }
  const float* ws_o = a.ws_o;
  const float* ws_lse = a.ws_lse;
  // The next kernel (usually the next step's append) may be scheduled at once: every kernel
  // of this library that can follow this one waits for its predecessor's grid before it
  // touches memory, and this grid completes only after its own wait below.  That hides the
  // successor's scheduling behind this merge.
  pdl_trigger();
  pdl_wait();  // the decode kernel's pieces must be complete
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float lse2 = -INFINITY;
  // online combine state; shared-prefix partials (normalised, weight 2^lse2) start it
  float M = -INFINITY, wsum = 0.f;
  for (int split = 0; pre_o && split < pre_splits; ++split) {
    const int64_t row = (int64_t)split * batch * hq + bh;
    const float l2 = pre_lse2[row];
    if (l2 == -INFINITY) continue;
    const float4 ov = reinterpret_cast<const float4*>(pre_o + row * kHeadDim)[lane];
    const float Mn = fmaxf(M, l2);
    const float fa = (M == -INFINITY) ? 0.f : fast_exp2(M - Mn);
    const float fb = fast_exp2(l2 - Mn);
    wsum = wsum * fa + fb;
    acc.x = acc.x * fa + fb * ov.x;
    acc.y = acc.y * fa + fb * ov.y;
    acc.z = acc.z * fa + fb * ov.z;
    acc.w = acc.w * fa + fb * ov.w;
    M = Mn;
  }
  if (c_lo <= c_hi) {
    // with fewer tiles than CTAs some CTAs own nothing and wrote no piece
    const bool maybe_empty = total < grid;
    auto empty_cta = [&](int c) {
      return maybe_empty && total * c / grid == total * (c + 1) / grid;
    };
    // online combine, four pieces per round: their lse and o are loaded together
    for (int c0 = c_lo; c0 <= c_hi; c0 += 4) {
      float lv[4];
      float4 ov[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = c0 + k;
        lv[k] = -INFINITY;
        ov[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c <= c_hi && !empty_cta(c)) {
          const int64_t slot = (unit + c) * 8 + hh;
          lv[k] = ws_lse[slot];
          ov[k] = reinterpret_cast<const float4*>(ws_o + slot * kHeadDim)[lane];
        }
      }
      const float mc = fmaxf(fmaxf(lv[0], lv[1]), fmaxf(lv[2], lv[3]));
      const float Mn = fmaxf(M, mc);
      if (Mn == -INFINITY) continue;
      const float corr = (M == -INFINITY) ? 0.f : fast_exp2(M - Mn);
      wsum *= corr;
      acc.x *= corr;
      acc.y *= corr;
      acc.z *= corr;
      acc.w *= corr;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float f = (lv[k] == -INFINITY) ? 0.f : fast_exp2(lv[k] - Mn);
        wsum += f;
        acc.x += f * ov[k].x;
        acc.y += f * ov[k].y;
        acc.z += f * ov[k].z;
        acc.w += f * ov[k].w;
      }
      M = Mn;
    }
  }
  if (M != -INFINITY) {
    const float inv = 1.f / wsum;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    lse2 = M + log2f(wsum);
  }
  uint2 pk;
  pk.x = pack_bf16x2(acc.x, acc.y);
  pk.y = pack_bf16x2(acc.z, acc.w);
  reinterpret_cast<uint2*>(a.out + bh * kHeadDim)[lane] = pk;
  if (a.lse && lane == 0) a.lse[bh] = lse2 * kLn2;
}

__global__ void visible_ranges_kernel(const int64_t* __restrict__ pos, int64_t batch, int32_t lp,
                                      int32_t w, int32_t* __restrict__ out) {
  const int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  const int64_t p = pos[b];
  VisibleRanges r{0, 0, 0, 0};
  if (p >= 0) r = visible_ranges(p, lp, w);
  out[b * 4 + 0] = r.pre_len;
  out[b * 4 + 1] = r.seg0_start;
  out[b * 4 + 2] = r.seg0_len;
  out[b * 4 + 3] = r.seg1_len;
}

int occupancy_per_sm() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  if (cached[dev] == 0) {
    int occ = 0;
    const size_t sb = smem_bytes(kStages);
    cudaFuncSetAttribute(decode_kernel<kStages, kPlain>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
    cudaFuncSetAttribute(decode_kernel<kStages, kReset>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
    // the grid must fit in one wave of whichever mode is launched: take the smaller
    int o[2] = {0, 0};
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o[0], decode_kernel<kStages, kPlain>,
                                                      kThreads, sb) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o[1], decode_kernel<kStages, kReset>,
                                                      kThreads, sb) != cudaSuccess)
      o[0] = o[1] = 1;
    occ = o[0] < o[1] ? o[0] : o[1];
    if (occ < 1) occ = 1;
    cached[dev] = occ < kCtasPerSm ? occ : kCtasPerSm;
  }
  return cached[dev];
}

// Stream-K grid size for this shape, or 0 for the per-unit schedule.  `force` selects
// stream-K whenever the batch fits its prefix table (the caller then always gets partials
// to merge, e.g. with a shared-prefix pass).
int64_t streamk_grid(int64_t batch, int32_t hkv, int64_t max_keys, bool force = false) {
  const int64_t units = batch * hkv;
  const int64_t slots = (int64_t)sm_count() * occupancy_per_sm();
  if (batch > kMaxStreamKSeqs || (units >= slots && !force)) return 0;
  const int64_t max_tiles = units * ((max_keys + kDecodeTile - 1) / kDecodeTile + 2);
  int64_t g = max_tiles / kMinTilesPerCta;
  // forced (prefix partials to fold in) with more units than CTA slots: about one unit per
  // CTA over several waves streams faster than one wave of long shares
  if (g > slots) g = (force && units > slots) ? units : slots;
  // a full wave: prefer a multiple of the unit count when one fills at least 5/6 of the
  // slots, so that with equally long units (every sequence past L_prefix + W) each share ends
  // on a unit boundary and no CTA switches unit mid-stream (batch 32 / 64 / 128 at W 4096:
  // 1.1-1.8, 0.5-1.6 and 0.5-1.1 us per step faster; with 200 of 296 slots, slower)
  if (!force && g == slots && units <= slots) {
    const int64_t ga = units * (slots / units);
    if (ga * 6 >= slots * 5) g = ga;
  }
  if (g < 1) g = 1;
  return g;
}

}  // namespace

int decode_splits(int64_t batch, int32_t hkv, int64_t max_keys) {
  const int64_t g = streamk_grid(batch, hkv, max_keys);
  return g > 0 ? static_cast<int>(g) : 1;
}

size_t decode_workspace_bytes(int64_t batch, int32_t hkv, int64_t max_keys, bool force_streamk) {
  const int64_t g = streamk_grid(batch, hkv, max_keys, force_streamk);
  if (g == 0) return 0;
  const size_t slots = size_t(batch * hkv + g) * 8;
  const size_t o_bytes = slots * kHeadDim * sizeof(float);
  const size_t lse_bytes = (slots * sizeof(float) + 255) & ~size_t(255);
  return o_bytes + lse_bytes;
}

int launch_decode(const DecodeLaunch& l, cudaStream_t stream) {
  const int group = l.hq / l.hkv;
  const int64_t max_keys =
      l.full_mode ? l.lmax : (int64_t)(l.lcap > l.lp ? l.lcap : l.lp) + l.w;
  const bool force = l.pre_o != nullptr;  // prefix partials are combined by the merge
  const int64_t g = streamk_grid(l.batch, l.hkv, max_keys, force);
  if (force && g == 0) return fail(PS_ERR_UNSUPPORTED, "shared-prefix decode needs batch <= 1024");
  if (g > 0 && l.workspace == nullptr)
    return fail(PS_ERR_WORKSPACE, "split-K decode launched without a workspace");
  const int64_t units = l.batch * l.hkv;
  // window-only decode reads no prefix rows: no prefix map (it may describe fewer units);
  // a prefix store with room for appended tokens has lcap rows per (sequence, KV head)
  const int32_t pre_rows = l.lcap > l.lp ? l.lcap : l.lp;
  const int32_t dim0 =
      l.full_mode ? static_cast<int32_t>(l.lmax) : (l.skip_prefix ? 0 : pre_rows);

  CUtensorMap mk0, mv0, mk1, mv1;
  if (l.paged) {
    // the pool [n_blocks][Hkv][64][D]: a 4-D map whose box is one half-row block
    const uint64_t dims[4] = {kHeadDim, (uint64_t)kDecodeTile, (uint64_t)l.hkv,
                              (uint64_t)l.n_blocks};
    const uint32_t box[4] = {64, (uint32_t)kDecodeTile, 1, 1};
    if (!make_map_4d(&mk0, l.k0, dims, box) || !make_map_4d(&mv0, l.v0, dims, box))
      return PS_ERR_CUDA;
    mk1 = mk0;
    mv1 = mv0;
  } else if (dim0 > 0) {
    if (!make_map_3d(&mk0, l.k0, kHeadDim, dim0, units, 64, kDecodeTile) ||
        !make_map_3d(&mv0, l.v0, kHeadDim, dim0, units, 64, kDecodeTile))
      return PS_ERR_CUDA;
  }
  if (!l.full_mode && !l.paged) {
    if (!make_map_3d(&mk1, l.k1, kHeadDim, l.w, units, 64, kDecodeTile) ||
        !make_map_3d(&mv1, l.v1, kHeadDim, l.w, units, 64, kDecodeTile))
      return PS_ERR_CUDA;
  }
  if (dim0 == 0 && !l.paged) {
    mk0 = mk1;
    mv0 = mv1;
  }
  if (l.full_mode) {
    mk1 = mk0;
    mv1 = mv0;
  }

  DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16*>(l.q);
  a.pos = l.pos;
  a.out = static_cast<__nv_bfloat16*>(l.out);
  a.lse = l.lse;
  const size_t nslots = size_t(units + g) * 8;
  a.ws_o = g ? static_cast<float*>(l.workspace) : nullptr;
  a.ws_lse = g ? a.ws_o + nslots * kHeadDim : nullptr;
  a.status = l.status;
  a.batch = static_cast<int32_t>(l.batch);
  a.hq = l.hq;
  a.hkv = l.hkv;
  a.group = group;
  a.lp = l.full_mode ? static_cast<int32_t>(l.lmax) : l.lp;
  a.w = l.full_mode ? 1 : l.w;
  a.dim0 = dim0;
  a.streamk = g > 0 ? 1 : 0;
  a.full_mode = l.full_mode;
  a.lmax = l.lmax;
  a.scale_log2 = l.scale * kLog2e;
  a.skip_prefix = l.skip_prefix;
  a.reset_pe = l.reset_pe;
  a.after_append = l.after_append;
  a.paged = l.paged;
  a.table = l.table;
  a.table_stride = l.table_stride;
  a.pre_blocks = (l.lp + kDecodeTile - 1) / kDecodeTile;
  a.n_blocks = l.n_blocks;
  a.pin_count = l.pin_count;
  a.pin_pos = l.pin_pos;
  a.pin_cap = (l.lcap > l.lp) ? l.lcap - l.lp : 0;
  for (int i = 0; i < kHeadDim / 2; ++i)
    a.inv_freq[i] = l.reset_pe ? pow(l.rope_theta, -2.0 * i / double(kHeadDim)) : 0.0;
  const int32_t pre_splits = l.pre_o ? (l.pre_splits > 0 ? l.pre_splits : 1) : 0;

  const size_t sb = smem_bytes(kStages);
  occupancy_per_sm();  // sets the shared-memory attribute once per device
  const int64_t grid = g > 0 ? g : units;
  if (grid <= 0) return PS_OK;
  if (grid > 0x7fffffff || l.batch > 0x7fffffff)
    return fail(PS_ERR_UNSUPPORTED, "decode grid too large");
  auto kern = a.reset_pe ? decode_kernel<kStages, kReset> : decode_kernel<kStages, kPlain>;
  int rc = check_cuda(launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(kThreads), sb,
                                 stream, mk0, mv0, mk1, mv1, a),
                      "decode_kernel launch");
  if (rc != PS_OK) return rc;
  if (l.before_merge) {
    rc = l.before_merge(l.before_merge_ctx, stream);
    if (rc != PS_OK) return rc;
  }
  if (g > 0) {
    rc = check_cuda(
        launch_pdl(merge_kernel, dim3(static_cast<unsigned>((l.batch * l.hq + 3) / 4)), dim3(128),
                   0, stream, a, static_cast<int32_t>(g), l.pre_o, l.pre_lse2, pre_splits),
        "merge_kernel launch");
  }
  return rc;
}

cudaError_t launch_visible_ranges(const int64_t* pos, int64_t batch, int32_t lp, int32_t w,
                                  int32_t* out, cudaStream_t stream) {
  if (batch <= 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((batch + 127) / 128);
  visible_ranges_kernel<<<blocks, 128, 0, stream>>>(pos, batch, lp, w, out);
  return cudaGetLastError();
}

// ------------------------------------------------- decode with built-in scratch
// Scratch for callers that cannot allocate device memory: the split-K partials of
// launch_decode_static_scratch live in this file-scope array.  It is part of the loaded
// module, so every GPU that loads the library holds it until the process exits.  All calls
// share it; it keeps the last call's contents (nothing in it has to start at zero), and
// calls that overlap on the GPU (for example on two streams) race on it.
static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {nullptr};
}  // namespace

int launch_decode_static_scratch(const DecodeLaunch& l, cudaStream_t stream) {
  const int64_t max_keys = l.full_mode ? l.lmax : (int64_t)l.lp + l.w;
  const size_t need = decode_workspace_bytes(l.batch, l.hkv, max_keys);
  if (need > kDecodeScratchBytes)
    return fail(PS_ERR_WORKSPACE,
                "decode needs " + std::to_string(need) + " bytes of scratch; the built-in array "
                "holds " + std::to_string(kDecodeScratchBytes) + " (use ps_decode_attn)");
  int dev = 0;
  int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
  if (rc != PS_OK) return rc;
  if (dev < 0 || dev >= 64) return fail(PS_ERR_UNSUPPORTED, "device index above 63");
  // Host code cannot use g_decode_scratch's address directly: on the host the name is a
  // stand-in.  The runtime is asked, with the device current, on every call made outside a
  // stream capture, so a context torn down and created again (cudaDeviceReset), which may
  // load the module at a new address, is never handed a stale pointer.  Inside a capture the
  // address recorded by the last call made outside one is used.
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
    cudaGetLastError();  // e.g. the legacy stream while another stream captures
    cs = cudaStreamCaptureStatusActive;
  }
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (cs == cudaStreamCaptureStatusNone || g_scratch_ptr[dev] == nullptr) {
      void* p = nullptr;
      rc = check_cuda(cudaGetSymbolAddress(&p, g_decode_scratch), "cudaGetSymbolAddress");
      if (rc != PS_OK) return rc;
      g_scratch_ptr[dev] = p;
    }
    ptr = g_scratch_ptr[dev];
  }
  DecodeLaunch l2 = l;
  l2.workspace = ptr;
  return launch_decode(l2, stream);
}

}  // namespace ps
