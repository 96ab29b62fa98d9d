// Split-K decode attention for the Prefix Sliding KV store (and the full-attention
// comparator over a linear cache), sm_100a.
//
// What it computes ("Prefix Sliding 完全拆解", §核心机制, eq. A(i)): the query of sequence b
// at position p attends only its visible keys, the prefix rows [0, min(p+1, Lp)) and the
// window positions [max(Lp, p+1-W), p+1), which live in ring slots (pos - Lp) mod W.  Only
// those rows are read ("§Kernel 实现": evicted keys are never loaded), so the bytes read per
// step stop growing once the window is full (eq. L_total).
//
// Design:
//  * One CTA per (sequence, KV head, split).  The visible keys are cut into 64-row TMA
//    tiles (see make_tiling); a split owns a contiguous run of tiles.
//  * Warp 4 is the producer: one lane issues four 3-D TMA loads per tile (K and V, two
//    64-column halves each, 128-byte swizzle) into a STAGES-deep mbarrier ring.
//  * Warps 0-3 consume 16 keys each per tile with warp-level bf16 tensor-core MMAs in fp32:
//      S^T[16 keys x 8 heads] = K[16 x 128] . Q^T       (GQA: the 8 query heads of the
//                                                          KV head share every K/V load)
//      O^T[128 x 8 heads]    += V^T[128 x 16] . P^T
//    P^T is moved from the accumulator layout to the operand layout with movmatrix.
//    Softmax runs online in base 2 with warp-shuffle max reductions.
//  * The four warps' (m, l, O) states are merged in shared memory; with one split the CTA
//    writes bf16 out (and lse) directly, otherwise normalised fp32 partials plus their
//    base-2 lse go to the workspace and merge_kernel combines them.
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
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kBoxBytes = kDecodeTile * 128;  // 64 rows x 64 bf16
constexpr int kTileBytes = 2 * kBoxBytes;     // one K (or V) tile: two column halves
constexpr int kStageBytes = 2 * kTileBytes;   // K + V
constexpr int kStages = 3;
constexpr int kMaxSplits = 64;
constexpr int kMinTilesPerSplit = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr size_t smem_bytes(int stages) { return 1024 + size_t(stages) * kStageBytes + 256; }

struct DecodeArgs {
  const __nv_bfloat16* q;
  const int64_t* pos;
  __nv_bfloat16* out;
  float* lse;
  float* ws_o;    // [units, splits, 8, D] normalised partial outputs
  float* ws_lse;  // [units, splits, 8] base-2 lse of each partial
  int32_t* status;
  int32_t hq, hkv, group;
  int32_t lp, w, dim0;
  int32_t splits, full_mode;
  int64_t lmax;
  float scale_log2;
};

// Offset of the 16-byte chunk `chunk` (0..7) of box row `row` under the 128-byte swizzle
// TMA applies (chunk index XOR row mod 8; boxes start 1024-byte aligned).
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return uint32_t(row) * 128u + (uint32_t(chunk ^ (row & 7)) << 4);
}

template <int STAGES>
__global__ void __launch_bounds__(kThreads)
    decode_kernel(const __grid_constant__ CUtensorMap mk0, const __grid_constant__ CUtensorMap mv0,
                  const __grid_constant__ CUtensorMap mk1, const __grid_constant__ CUtensorMap mv1,
                  const DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * kStageBytes);
  uint64_t* empty = full + STAGES;

  const int split = blockIdx.x % a.splits;
  const int unit = blockIdx.x / a.splits;  // b * hkv + h
  const int b = unit / a.hkv;
  const int h = unit % a.hkv;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int64_t p = a.pos[b];
  const bool bad = (p < 0) || (a.full_mode && p >= a.lmax);
  if (bad && threadIdx.x == 0 && split == 0 && a.status)
    atomicOr(a.status, p < 0 ? PS_DEV_BAD_POS : PS_DEV_POS_RANGE);

  VisibleRanges r{0, 0, 0, 0};
  if (!bad) {
    if (a.full_mode) {
      r.pre_len = static_cast<int32_t>(p + 1);
    } else {
      r = visible_ranges(p, a.lp, a.w);
    }
  }
  const DecodeTiling t = make_tiling(r, a.dim0, a.w);
  const int t_begin = static_cast<int>((int64_t)t.total * split / a.splits);
  const int t_end = static_cast<int>((int64_t)t.total * (split + 1) / a.splits);
  const int ntiles = t_end - t_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  float o[8][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && ntiles > 0) {
      prefetch_tensormap(&mk0);
      prefetch_tensormap(&mv0);
      prefetch_tensormap(&mk1);
      prefetch_tensormap(&mv1);
      const uint64_t pol = l2_policy_evict_first();
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (i >= STAGES && !mbar_wait(&empty[s], ph ^ 1, a.status)) break;
        const DecodeTile d = tiling_tile(t, t_begin + i);
        const CUtensorMap* mk = d.map_id ? &mk1 : &mk0;
        const CUtensorMap* mv = d.map_id ? &mv1 : &mv0;
        uint8_t* st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        tma_load_3d_hint(st, mk, 0, d.row0, unit, &full[s], pol);
        tma_load_3d_hint(st + kBoxBytes, mk, 64, d.row0, unit, &full[s], pol);
        tma_load_3d_hint(st + kTileBytes, mv, 0, d.row0, unit, &full[s], pol);
        tma_load_3d_hint(st + kTileBytes + kBoxBytes, mv, 64, d.row0, unit, &full[s], pol);
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
    uint32_t qf[8][2];
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
    const float sl2 = a.scale_log2;
    const int arow = 16 * warp + (lane & 15);        // ldmatrix row for K
    const int achunk = lane >> 4;                    // 0/1: k 0-7 or 8-15
    const int vkey = 16 * warp + (lane & 7) + ((lane >> 4) << 3);
    const int vdoff = ((lane >> 3) & 1) << 3;
    const int r0 = 16 * warp + (lane >> 2);
    const int r1 = r0 + 8;

    for (int i = 0; i < ntiles; ++i) {
      const int s = i % STAGES;
      // warp-uniform outcome: ldmatrix / mma.sync below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / STAGES) & 1, a.status))) break;
      const DecodeTile d = tiling_tile(t, t_begin + i);
      const uint32_t kbase = smem_u32(smem + s * kStageBytes);
      const uint32_t vbase = kbase + kTileBytes;

      float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a0, a1, a2, a3;
        const uint32_t addr =
            kbase + (ks >> 2) * kBoxBytes + swz(arow, ((ks & 3) << 1) + achunk);
        ldmatrix_x4(addr, a0, a1, a2, a3);
        mma_bf16_16816(sc, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
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
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int dd = 16 * j + vdoff;
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(vbase + (dd >> 6) * kBoxBytes + swz(vkey, (dd & 63) >> 3), a0, a1, a2,
                          a3);
        mma_bf16_16816(o[j], a0, a1, a2, a3, b0, b1);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
  }
  __syncthreads();  // every tile consumed and every copy landed: stages are free

  // ---------------------------------------------- merge the four warps' states
  float* red_m = reinterpret_cast<float*>(smem);         // [4][8]
  float* red_l = red_m + kConsumerWarps * 8;             // [4][8]
  float* red_o = red_l + kConsumerWarps * 8;             // [4][8][D]
  if (warp < kConsumerWarps) {
    const int qq = lane & 3;
    if (lane < 4) {
      red_m[warp * 8 + 2 * qq] = m0;
      red_m[warp * 8 + 2 * qq + 1] = m1;
      red_l[warp * 8 + 2 * qq] = l0;
      red_l[warp * 8 + 2 * qq + 1] = l1;
    }
    float* ow = red_o + warp * 8 * kHeadDim;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int dlo = 16 * j + (lane >> 2);
      ow[(2 * qq) * kHeadDim + dlo] = o[j][0];
      ow[(2 * qq + 1) * kHeadDim + dlo] = o[j][1];
      ow[(2 * qq) * kHeadDim + dlo + 8] = o[j][2];
      ow[(2 * qq + 1) * kHeadDim + dlo + 8] = o[j][3];
    }
  }
  __syncthreads();
  if (threadIdx.x < kHeadDim) {
    const int dcol = threadIdx.x;
    for (int hh = 0; hh < a.group; ++hh) {
      float M = -INFINITY;
#pragma unroll
      for (int wv = 0; wv < kConsumerWarps; ++wv) M = fmaxf(M, red_m[wv * 8 + hh]);
      float oval = 0.f, lse2 = -INFINITY;
      if (M != -INFINITY) {
        float wsum = 0.f, osum = 0.f;
#pragma unroll
        for (int wv = 0; wv < kConsumerWarps; ++wv) {
          const float f = fast_exp2(red_m[wv * 8 + hh] - M);
          wsum += f * red_l[wv * 8 + hh];
          osum += f * red_o[(wv * 8 + hh) * kHeadDim + dcol];
        }
        oval = osum / wsum;
        lse2 = M + log2f(wsum);
      }
      const int head = h * a.group + hh;
      if (a.splits == 1) {
        a.out[((int64_t)b * a.hq + head) * kHeadDim + dcol] = __float2bfloat16_rn(oval);
        if (a.lse && dcol == 0) a.lse[(int64_t)b * a.hq + head] = lse2 * kLn2;
      } else {
        const int64_t slot = ((int64_t)unit * a.splits + split) * 8 + hh;
        a.ws_o[slot * kHeadDim + dcol] = oval;
        if (dcol == 0) a.ws_lse[slot] = lse2;
      }
    }
  }
}

// Combines the splits of one (sequence, query head): weights 2^(lse_s - max).
__global__ void __launch_bounds__(128)
    merge_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_lse,
                 __nv_bfloat16* __restrict__ out, float* __restrict__ lse, int32_t hq,
                 int32_t hkv, int32_t group, int32_t splits) {
  const int bh = blockIdx.x;
  const int b = bh / hq, head = bh % hq;
  const int h = head / group, hh = head % group;
  const int64_t unit = (int64_t)b * hkv + h;
  const int dcol = threadIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, ws_lse[(unit * splits + s) * 8 + hh]);
  float oval = 0.f, lse2 = -INFINITY;
  if (M != -INFINITY) {
    float wsum = 0.f, osum = 0.f;
    for (int s = 0; s < splits; ++s) {
      const int64_t slot = (unit * splits + s) * 8 + hh;
      const float f = fast_exp2(ws_lse[slot] - M);
      wsum += f;
      osum += f * ws_o[slot * kHeadDim + dcol];
    }
    oval = osum / wsum;
    lse2 = M + log2f(wsum);
  }
  out[(int64_t)bh * kHeadDim + dcol] = __float2bfloat16_rn(oval);
  if (lse && dcol == 0) lse[bh] = lse2 * kLn2;
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
    cudaFuncSetAttribute(decode_kernel<kStages>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)sb);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel<kStages>, kThreads, sb) !=
            cudaSuccess ||
        occ < 1)
      occ = 1;
    cached[dev] = occ;
  }
  return cached[dev];
}

}  // namespace

int decode_splits(int64_t batch, int32_t hkv, int64_t max_keys) {
  const int64_t units = batch * hkv;
  const int64_t slots = (int64_t)sm_count() * occupancy_per_sm();
  // enough CTAs to keep every SM streaming, never fewer than kMinTilesPerSplit tiles each
  const int64_t max_tiles = (max_keys + kDecodeTile - 1) / kDecodeTile + 2;
  int64_t s = units >= slots ? 1 : slots / units;
  const int64_t cap = max_tiles / kMinTilesPerSplit;
  if (s > cap) s = cap;
  if (s > kMaxSplits) s = kMaxSplits;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

size_t decode_workspace_bytes(int64_t batch, int32_t hkv, int64_t max_keys) {
  const int s = decode_splits(batch, hkv, max_keys);
  if (s <= 1) return 0;
  const size_t slots = size_t(batch) * hkv * s * 8;
  return slots * (kHeadDim + 1) * sizeof(float);
}

int launch_decode(const DecodeLaunch& l, cudaStream_t stream) {
  const int group = l.hq / l.hkv;
  const int64_t max_keys = l.full_mode ? l.lmax : (int64_t)l.lp + l.w;
  const int splits = decode_splits(l.batch, l.hkv, max_keys);
  const int64_t units = l.batch * l.hkv;
  const int32_t dim0 = l.full_mode ? static_cast<int32_t>(l.lmax) : l.lp;

  CUtensorMap mk0, mv0, mk1, mv1;
  // A zero-row tensor cannot be described; such a map is never used (no tiles), so it
  // borrows the other map.
  if (dim0 > 0) {
    if (!make_map_3d(&mk0, l.k0, kHeadDim, dim0, units, 64, kDecodeTile) ||
        !make_map_3d(&mv0, l.v0, kHeadDim, dim0, units, 64, kDecodeTile))
      return PS_ERR_CUDA;
  }
  if (!l.full_mode) {
    if (!make_map_3d(&mk1, l.k1, kHeadDim, l.w, units, 64, kDecodeTile) ||
        !make_map_3d(&mv1, l.v1, kHeadDim, l.w, units, 64, kDecodeTile))
      return PS_ERR_CUDA;
  }
  if (dim0 == 0) {
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
  const size_t nslots = size_t(units) * splits * 8;
  a.ws_o = static_cast<float*>(l.workspace);
  a.ws_lse = a.ws_o ? a.ws_o + nslots * kHeadDim : nullptr;
  a.status = l.status;
  a.hq = l.hq;
  a.hkv = l.hkv;
  a.group = group;
  a.lp = l.full_mode ? static_cast<int32_t>(l.lmax) : l.lp;
  a.w = l.full_mode ? 1 : l.w;
  a.dim0 = dim0;
  a.splits = splits;
  a.full_mode = l.full_mode;
  a.lmax = l.lmax;
  a.scale_log2 = l.scale * kLog2e;

  const size_t sb = smem_bytes(kStages);
  occupancy_per_sm();  // sets the shared-memory attribute once per device
  const int64_t grid = units * splits;
  if (grid <= 0) return PS_OK;
  if (grid > 0x7fffffff) return fail(PS_ERR_UNSUPPORTED, "decode grid too large");
  decode_kernel<kStages><<<static_cast<unsigned>(grid), kThreads, sb, stream>>>(mk0, mv0, mk1, mv1,
                                                                             a);
  int rc = check_cuda(cudaGetLastError(), "decode_kernel launch");
  if (rc != PS_OK) return rc;
  if (splits > 1) {
    merge_kernel<<<static_cast<unsigned>(l.batch * l.hq), kHeadDim, 0, stream>>>(
        a.ws_o, a.ws_lse, a.out, a.lse, l.hq, l.hkv, group, splits);
    rc = check_cuda(cudaGetLastError(), "merge_kernel launch");
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
  void* ptr = nullptr;
  {
    // Host code cannot use g_decode_scratch's address directly: on the host the name is a
    // stand-in.  Ask the runtime once per device, with that device current.
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
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
