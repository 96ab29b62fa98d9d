// Masked prefill / truncated-backprop context forward on 5th-generation tensor cores
// (tcgen05 + TMEM + TMA), sm_100a.
//
// What it computes ("Prefix Sliding 完全拆解", §核心机制 eq. A(i); §截断回传): for every row i
// of the sequence, softmax(q_i . k_j * scale) over the visible keys j in
// [0, min(Lp, i+1)) U [max(Lp, i-W+1), i] (sequence indices), times V.  Two-level filtering
// (§Kernel 实现): the device planner lists, per 128-row query tile, only the 128-key tiles
// that hold a visible pair; SKIP tiles are never loaded or multiplied.  FULL tiles run
// unmasked; PARTIAL tiles (the diagonal, the window's lower edge, the prefix's end and the
// ragged tail) get an element-wise mask.
//
// One CTA per (batch, query head, query tile), heaviest query tiles first, 6 warps:
//   warp 4  - TMA producer: the Q tile once, then K and V tiles of the plan into a
//             two-stage mbarrier ring (4-D tensor maps, 128-byte swizzle).
//   warp 5  - allocates 512 TMEM columns; one lane issues the MMAs:
//               S[buf] = Q K^T           (tcgen05.mma kind::f16, A and B from smem)
//               O     += P V             (A = P from TMEM, B = V from smem, MN-major)
//             and commits them to mbarriers.  S of tile j+1 is issued before PV of tile j,
//             so the tensor pipe computes the next scores while softmax runs.
//   warps 0-3 - softmax: thread r owns row r (TMEM lane r).  It reads its S row, masks it
//             on PARTIAL tiles, keeps the running max m and sum l in fp32 (base 2), writes
//             P as bf16 over the first 64 columns of the same S buffer, and signals the
//             MMA warp.  O is rescaled in TMEM only when the max of some row of the warp
//             grows by more than 8 (log2 units); otherwise P stays below 2^8 and the
//             stale max keeps fp32 sums exact enough.  The decision is warp-uniform
//             because tcgen05.ld/st are warp-collective.
//   Epilogue: the softmax warps read O, divide by l, store bf16 out and the natural-log lse.
// TMEM columns: S0 [0,128), S1 [128,256), O [256,384).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "ps_device.cuh"
#include "ps_internal.h"
#include "ps_ranges.cuh"

namespace ps {
namespace {

constexpr int kBq = kPrefillBq;
constexpr int kBk = kPrefillBk;
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 6 * 32;
constexpr int kKVStages = 2;
constexpr int kBoxBytes = 128 * 128;        // [128 rows][64 bf16]
constexpr int kTileBytes = 2 * kBoxBytes;   // [128 rows][128 bf16]
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t col_s(int s) { return s ? 128u : 0u; }
constexpr uint32_t kColO = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

constexpr size_t kSmemBytes = 1024 + kTileBytes * (1 + 2 * kKVStages) + 256;

struct PrefillArgs {
  const int32_t* off;  // [nq + 1] plan offsets
  const int32_t* ent;  // [n][2] (k_tile, flag)
  __nv_bfloat16* out;  // [B, S, Hq, D]
  float* lse;          // [B, Hq, S] or null
  int32_t* status;
  int64_t seq;
  int32_t batch, hq, group, nq;
  int32_t lp, w;
  float scale_log2;
};

__device__ __forceinline__ bool visible(int64_t row, int64_t col, int64_t seq, int32_t lp,
                                        int32_t w) {
  return col <= row && col < seq && (col < lp || col > row - w);
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                   const __grid_constant__ CUtensorMap mv, const PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kTileBytes;
  uint8_t* sV = sK + kKVStages * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kKVStages * kTileBytes);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* p_ready = bars + 7;   // [2]
  uint64_t* pv_done = bars + 9;
  uint64_t* mma_done = bars + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);

  const int64_t bh = (int64_t)a.batch * a.hq;
  const int qt = a.nq - 1 - static_cast<int>(blockIdx.x / bh);
  const int rem = static_cast<int>(blockIdx.x % bh);
  const int head = rem % a.hq;
  const int b = rem / a.hq;
  const int kvh = head / a.group;
  const int e0 = a.off[qt];
  const int n = a.off[qt + 1] - e0;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_ready[s], kSoftmaxWarps);
    }
    mbar_init(pv_done, 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&mq);
      prefetch_tensormap(&mk);
      prefetch_tensormap(&mv);
      mbar_arrive_expect_tx(q_full, kTileBytes);
      tma_load_4d(sQ, &mq, 0, head, qt * kBq, b, q_full);
      tma_load_4d(sQ + kBoxBytes, &mq, 64, head, qt * kBq, b, q_full);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int s = j & 1;
        if (j >= 2 && !mbar_wait(&kv_empty[s], ((j >> 1) & 1) ^ 1, a.status)) break;
        const int kt = a.ent[2 * (e0 + j)];
        mbar_arrive_expect_tx(&kv_full[s], 2 * kTileBytes);
        uint8_t* k_dst = sK + s * kTileBytes;
        uint8_t* v_dst = sV + s * kTileBytes;
        tma_load_4d(k_dst, &mk, 0, kvh, kt * kBk, b, &kv_full[s]);
        tma_load_4d(k_dst + kBoxBytes, &mk, 64, kvh, kt * kBk, b, &kv_full[s]);
        tma_load_4d(v_dst, &mv, 0, kvh, kt * kBk, b, &kv_full[s]);
        tma_load_4d(v_dst + kBoxBytes, &mv, 64, kvh, kt * kBk, b, &kv_full[s]);
        issued = j + 1;
      }
      // every issued copy lands before the CTA may exit
      mbar_wait(q_full, 0, a.status);
      for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j)
        mbar_wait(&kv_full[j & 1], (j >> 1) & 1, a.status);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(128, 128, false);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 128, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV);
      bool ok = mbar_wait(q_full, 0, a.status);
      auto issue_pv = [&](int i) -> bool {
        const int s = i & 1;
        if (!mbar_wait(&p_ready[s], (i >> 1) & 1, a.status)) return false;
        tc_fence_after();
        const uint32_t vb = v_addr + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // B = V[16 keys][128 d]: MN-major, 64-column halves 16 KB apart (LBO), 8-key
          // groups 1024 B apart (SBO); 16 keys = 2048 B per step.
          const uint64_t bdesc = umma_desc_sw128(vb + kk * 2048, kBoxBytes, 1024);
          umma_ts(tmem + kColO, tmem + col_s(s) + kk * 8, bdesc, idesc_pv,
                  (i > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&kv_empty[s]);
        umma_commit(pv_done);
        return true;
      };
      for (int j = 0; ok && j < n; ++j) {
        const int s = j & 1;
        if (!mbar_wait(&kv_full[s], (j >> 1) & 1, a.status)) {
          ok = false;
          break;
        }
        // S buffer s held P_{j-2}: PV_{j-2} must have finished reading it
        if (j >= 2 && !mbar_wait(pv_done, (j - 2) & 1, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kb = k_addr + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // A = Q, B = K: K-major, 128-byte rows, 8-row groups 1024 B apart; 16 columns =
          // 32 B per step inside a 64-column half.
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          umma_ss(tmem + col_s(s), umma_desc_sw128(q_addr + off, 16, 1024),
                  umma_desc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[s]);
        if (j >= 1 && !issue_pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && n > 0) issue_pv(n - 1);
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, a.status);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroup
    const int r = threadIdx.x;  // row within the tile == TMEM lane
    const int64_t row = (int64_t)qt * kBq + r;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = a.scale_log2;
    float m = -INFINITY;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int s = j & 1;
      const int kt = a.ent[2 * (e0 + j)];
      const int flag = a.ent[2 * (e0 + j) + 1];
      // warp-uniform outcome: the tcgen05.ld/st below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[s], (j >> 1) & 1, a.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t raw[32];
        tmem_ld32(lane_base + col_s(s) + 32 * c, raw);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) x[32 * c + i] = __uint_as_float(raw[i]) * sl2;
      }
      if (flag == PS_TILE_PARTIAL) {
        const int64_t k0 = (int64_t)kt * kBk;
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (!visible(row, k0 + i, a.seq, a.lp, a.w)) x[i] = -INFINITY;
      }
      float mt = x[0];
#pragma unroll
      for (int i = 1; i < 128; ++i) mt = fmaxf(mt, x[i]);
      const float m_new = fmaxf(m, mt);
      // The rescale touches TMEM with warp-collective tcgen05.ld/st, so the decision is
      // taken per warp: if any row of the warp needs it, every row of the warp rescales
      // (exact for every row, since m_new >= m).
      if (__any_sync(0xffffffffu, m_new > m + kRescaleThreshold)) {
        float f = 1.f;
        if (m_new != -INFINITY) f = (m == -INFINITY) ? 0.f : fast_exp2(m - m_new);
        if (j > 0) {
          // O holds PV_0..PV_{j-1}; wait for the last of them, then scale in place
          if (!__all_sync(0xffffffffu, mbar_wait(pv_done, (j - 1) & 1, a.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + kColO + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st32(lane_base + kColO + 32 * c, o);
          }
          tmem_wait_st();
        }
        l *= f;
        if (m_new != -INFINITY) m = m_new;
      }
      const float mref = (m == -INFINITY) ? 0.f : m;
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = fast_exp2(x[32 * c + 2 * i] - mref);
          const float p1 = fast_exp2(x[32 * c + 2 * i + 1] - mref);
          sum += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(lane_base + col_s(s) + 16 * c, pk);
      }
      l += sum;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[s]);
    }
    // ------------------------------------------------------------ epilogue
    if (ok && n > 0 && __all_sync(0xffffffffu, mbar_wait(pv_done, (n - 1) & 1, a.status))) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const bool store = row < a.seq;
      __nv_bfloat16* orow = a.out + (((int64_t)b * a.seq + row) * a.hq + head) * kHeadDim;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(lane_base + kColO + 32 * c, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l,
                              __uint_as_float(o[2 * i + 1]) * inv_l);
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if (store && a.lse)
        a.lse[((int64_t)b * a.hq + head) * a.seq + row] =
            l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t prefill_workspace_bytes(int64_t seq, int32_t lp, int32_t w) {
  return prefill_plan_bytes(seq, prefill_plan_tiles(seq, lp, w));
}

int launch_prefill(const PrefillLaunch& l, cudaStream_t stream) {
  const int64_t nq = (l.seq + kBq - 1) / kBq;
  const int group = l.hq / l.hkv;
  // plan into the workspace (and the caller's copy)
  int rc = check_cuda(launch_plan(l.seq, l.lp, l.w, l.n_tiles, l.workspace, l.plan_out, stream),
                      "plan_kernel launch");
  if (rc != PS_OK) return rc;

  CUtensorMap mq, mk, mv;
  const uint64_t dq[4] = {kHeadDim, (uint64_t)l.hq, (uint64_t)l.seq, (uint64_t)l.batch};
  const uint64_t dk[4] = {kHeadDim, (uint64_t)l.hkv, (uint64_t)l.seq, (uint64_t)l.batch};
  const uint32_t box[4] = {64, 1, 128, 1};
  if (!make_map_4d(&mq, l.q, dq, box) || !make_map_4d(&mk, l.k, dk, box) ||
      !make_map_4d(&mv, l.v, dk, box))
    return PS_ERR_CUDA;

  PrefillArgs a;
  a.off = static_cast<const int32_t*>(l.workspace);
  a.ent = reinterpret_cast<const int32_t*>(static_cast<const char*>(l.workspace) +
                                           align256(size_t(nq + 1) * 4));
  a.out = static_cast<__nv_bfloat16*>(l.out);
  a.lse = l.lse;
  a.status = l.status;
  a.seq = l.seq;
  a.batch = static_cast<int32_t>(l.batch);
  a.hq = l.hq;
  a.group = group;
  a.nq = static_cast<int32_t>(nq);
  a.lp = l.lp;
  a.w = l.w;
  a.scale_log2 = l.scale * kLog2e;

  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    rc = check_cuda(cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes),
                    "cudaFuncSetAttribute(prefill_kernel)");
    if (rc != PS_OK) return rc;
    attr_set[dev] = true;
  }
  const int64_t grid = l.batch * l.hq * nq;
  if (grid <= 0) return PS_OK;
  if (grid > 0x7fffffffLL) return fail(PS_ERR_UNSUPPORTED, "prefill grid too large");
  prefill_kernel<<<static_cast<unsigned>(grid), kThreads, kSmemBytes, stream>>>(mq, mk, mv, a);
  return check_cuda(cudaGetLastError(), "prefill_kernel launch");
}

}  // namespace ps
