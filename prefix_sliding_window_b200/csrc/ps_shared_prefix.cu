// Shared-prefix decode: the prefix pass, on 5th-generation tensor cores, sm_100a.
//
// When groups of sequences decode from one prompt ("Prefix Sliding 完全拆解", §Kernel 实现:
// the sampling code passes one prompt text per request, and the accuracy tables average many
// samples per problem), every sequence of a group pins the same L_prefix rows (§核心机制,
// eq. A(i)).  Plain decode streams those rows once per sequence; here they are streamed once
// per group: the queries of all (sequence, query head) pairs of a group that share a KV head
// form the rows of one matrix, so each 128-key prefix tile feeds a 128 x 128 tensor-core
// product instead of 8 query columns.  The pass writes, per (sequence, query head), the
// normalised attention over the prefix rows [0, min(pos + 1, L_prefix)) and its base-2
// log-sum-exp; the window-only decode folds it in (log-sum-exp weighted), which gives exactly
// the attention over the prefix and the window together.
//
// One CTA per (group, KV head, 128-row block of that group's query rows, key-range split):
// row r is sequence r / g of the group, query head h * g + r % g; each split covers a run
// of 128-key prefix tiles and writes its own partial, so few groups still fill the GPU.
// 6 warps:
//   all     - stage the query block into shared memory (128-byte swizzled, K-major);
//   warp 4  - TMA producer: K and V prefix tiles (128 rows, two 64-column halves) into a
//             2-stage ring;
//   warp 5  - allocates TMEM, issues S[buf] = Q K^T one tile ahead and O += P V (A = P from
//             TMEM, B = V MN-major);
//   warps 0-3 - one row each: masks keys past the row's visible prefix, online softmax in
//             base 2 (O rescaled in TMEM only when a row's max grows by more than 2^8), P as
//             bf16 over S, and the epilogue.
// TMEM columns: S0 [0,128), S1 [128,256), O [256,384).

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "ps_device.cuh"
#include "ps_internal.h"

namespace ps {
namespace {

constexpr int kSpThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kBoxBytes = 128 * 128;       // [128 rows][64 bf16]
constexpr int kTileBytes = 2 * kBoxBytes;  // [128 rows][128 bf16]
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr float kRescaleThreshold = 8.f;  // log2 units
constexpr float kLog2e = 1.4426950408889634f;
constexpr size_t kSpSmem = 1024 + size_t(kTileBytes) * (1 + 2 * kStages) + 256;

struct SpArgs {
  const __nv_bfloat16* q;
  const int64_t* pos;
  float* o;
  float* lse2;
  int32_t* status;
  int32_t hq, hkv, group, gsize;
  int32_t lp, nkt, row_tiles;
  int32_t splits, per;  // key-range splits of the prefix and tiles per split
  int64_t split_rows;   // batch * Hq: stride between the splits' partials
  float scale_log2;
};

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__global__ void __launch_bounds__(kSpThreads, 1)
    shared_prefix_kernel(const __grid_constant__ CUtensorMap mk,
                         const __grid_constant__ CUtensorMap mv, const SpArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kTileBytes;          // [kStages]
  uint8_t* sV = sK + kStages * kTileBytes;  // [kStages]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kStages * kTileBytes);
  uint64_t* kv_full = bars;       // [2]
  uint64_t* kv_empty = bars + 2;  // [2]
  uint64_t* s_full = bars + 4;    // [2]
  uint64_t* p_ready = bars + 6;   // [2]
  uint64_t* pv_done = bars + 8;   // [2]
  uint64_t* o_full = bars + 10;
  uint64_t* mma_done = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);

  // block = (group, KV head, row block, key split); the split owns prefix tiles
  // [kt0, kt0 + n), tile indices below are relative to kt0
  const int split = blockIdx.x % a.splits;
  const int item = blockIdx.x / a.splits;
  const int kt0 = split * a.per;
  const int n = (a.nkt - kt0 < a.per) ? a.nkt - kt0 : a.per;
  const int t = item % a.row_tiles;
  const int rest = item / a.row_tiles;
  const int h = rest % a.hkv;
  const int grp = rest / a.hkv;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_rows = a.gsize * a.group;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_ready[s], 4);
      mbar_init(&pv_done[s], 1);
    }
    mbar_init(o_full, 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensormap(&mk);
    prefetch_tensormap(&mv);
  }
  pdl_wait();  // q, positions and the prefix come from earlier kernels
  pdl_trigger();

  // query block: 128 rows x 16 chunks of 16 bytes, K-major, 128-byte swizzle
  for (int c = threadIdx.x; c < 128 * 16; c += kSpThreads) {
    const int r = c >> 4, ch = c & 15;
    const int rr = t * 128 + r;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (rr < n_rows) {
      const int64_t b = (int64_t)grp * a.gsize + rr / a.group;
      const int head = h * a.group + rr % a.group;
      v = *reinterpret_cast<const uint4*>(a.q + (b * a.hq + head) * kHeadDim + ch * 8);
    }
    const int half = ch >> 3, cc = ch & 7;
    *reinterpret_cast<uint4*>(sQ + half * kBoxBytes + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
  }
  fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      const int unit = grp * a.hkv + h;
      int issued = 0;
      for (int kt = 0; kt < n; ++kt) {
        const int s = kt & 1;
        if (kt >= 2 && !mbar_wait(&kv_empty[s], static_cast<uint32_t>(((kt >> 1) - 1) & 1),
                                  a.status))
          break;
        mbar_arrive_expect_tx(&kv_full[s], 2 * kTileBytes);
        uint8_t* k = sK + s * kTileBytes;
        uint8_t* v = sV + s * kTileBytes;
        const int row0 = (kt0 + kt) * 128;
        tma_load_3d(k, &mk, 0, row0, unit, &kv_full[s]);
        tma_load_3d(k + kBoxBytes, &mk, 64, row0, unit, &kv_full[s]);
        tma_load_3d(v, &mv, 0, row0, unit, &kv_full[s]);
        tma_load_3d(v + kBoxBytes, &mv, 64, row0, unit, &kv_full[s]);
        issued = kt + 1;
      }
      for (int kt = (issued > 2 ? issued - 2 : 0); kt < issued; ++kt)
        mbar_wait(&kv_full[kt & 1], static_cast<uint32_t>((kt >> 1) & 1), a.status);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(128, 128, false);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 128, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      bool ok = true;
      auto issue_s = [&](int kt) {
        const int s = kt & 1;
        if (!mbar_wait(&kv_full[s], static_cast<uint32_t>((kt >> 1) & 1), a.status) ||
            (kt >= 2 &&
             !mbar_wait(&pv_done[s], static_cast<uint32_t>(((kt >> 1) - 1) & 1), a.status))) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint32_t kb = k_addr + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          umma_ss(tmem + 128u * s, umma_desc_sw128(q_addr + off, 16, 1024),
                  umma_desc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[s]);
      };
      if (n > 0) issue_s(0);
      for (int kt = 0; ok && kt < n; ++kt) {
        if (kt + 1 < n) issue_s(kt + 1);  // next scores while this tile's softmax runs
        if (!ok) break;
        const int s = kt & 1;
        if (!mbar_wait(&p_ready[s], static_cast<uint32_t>((kt >> 1) & 1), a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t vb = v_addr + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // B = V[16 keys][128 d], MN-major: halves 16 KB apart (LBO), 8-key groups 1024 B
          const uint64_t bdesc = umma_desc_sw128(vb + kk * 2048, kBoxBytes, 1024);
          umma_ts(tmem + kColO, tmem + 128u * s + kk * 8, bdesc, idesc_pv,
                  (kt > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&pv_done[s]);
        umma_commit(&kv_empty[s]);
      }
      if (ok) umma_commit(o_full);
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, a.status);
    }
  } else {
    // ---------------------------------------------------------------- softmax rows
    const int r = threadIdx.x;  // TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int rr = t * 128 + r;
    const bool valid = rr < n_rows;
    int64_t b = 0;
    int head = 0;
    int64_t kvis = 0;  // visible prefix rows of this query
    if (valid) {
      b = (int64_t)grp * a.gsize + rr / a.group;
      head = h * a.group + rr % a.group;
      const int64_t p = a.pos[b];
      if (p >= 0) kvis = p + 1 < a.lp ? p + 1 : a.lp;
    }
    const float sl2 = a.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int kt = 0; kt < n; ++kt) {
      const int s = kt & 1;
      ok = ok && __all_sync(0xffffffffu,
                            mbar_wait(&s_full[s], static_cast<uint32_t>((kt >> 1) & 1), a.status));
      if (!ok) break;
      tc_fence_after();
      float x[128];
      {
        uint32_t raw[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + 128u * s + 32 * c, raw[c]);
        tmem_wait_ld();
        const int64_t lim = kvis - (int64_t)(kt0 + kt) * 128;  // visible columns [0, lim)
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            x[32 * c + i] = (32 * c + i < lim) ? __uint_as_float(raw[c][i]) * sl2 : -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 128; i += 2) mx = max3f(mx, x[i], x[i + 1]);
      const float m_new = fmaxf(m, mx);
      if (__any_sync(0xffffffffu, m_new - m > kRescaleThreshold)) {
        float f = 1.f;
        if (m_new != -INFINITY) f = (m == -INFINITY) ? 0.f : fast_exp2(m - m_new);
        if (kt > 0) {
          // O holds the PVs of tiles < kt: wait for the last, then scale in place
          const int sp = (kt - 1) & 1;
          if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[sp],
                                                 static_cast<uint32_t>(((kt - 1) >> 1) & 1),
                                                 a.status))) {
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
      const float ms = (m == -INFINITY) ? 0.f : m;
      uint32_t pk[64];
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float p0 = fast_exp2(x[2 * i] - ms), p1 = fast_exp2(x[2 * i + 1] - ms);
        acc += p0 + p1;
        pk[i] = cvt_bf16x2(p0, p1);
      }
      l += acc;
      // P over the first 64 columns of this row's own S buffer
      tmem_st32(lane_base + 128u * s, *reinterpret_cast<uint32_t(*)[32]>(pk));
      tmem_st32(lane_base + 128u * s + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[s]);
    }
    // epilogue: normalised prefix attention and its base-2 lse.  The TMEM loads are
    // warp-collective, so every lane runs them; only rows of the group are stored.
    const bool fin = __all_sync(0xffffffffu,
                                ok && (n == 0 || mbar_wait(o_full, 0, a.status)));
    if (fin) {
      const int64_t orow = split * a.split_rows + b * a.hq + head;
      float* dst = a.o + orow * kHeadDim;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      if (n > 0) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColO + 32 * c, o);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              reinterpret_cast<float4*>(dst + 32 * c)[v] = make_float4(
                  __uint_as_float(o[4 * v]) * inv, __uint_as_float(o[4 * v + 1]) * inv,
                  __uint_as_float(o[4 * v + 2]) * inv, __uint_as_float(o[4 * v + 3]) * inv);
          }
        }
      } else if (valid) {
        for (int v = 0; v < 32; ++v)
          reinterpret_cast<float4*>(dst)[v] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (valid) a.lse2[orow] = l > 0.f ? m + log2f(l) : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

// Enough key-range splits that the blocks cover every SM once (each split keeps at least
// one 128-key tile); the window pass and the merge fold the splits' partials together.
int shared_prefix_splits(int64_t batch, int64_t gsize, int32_t hq, int32_t hkv, int32_t lp) {
  const int64_t rows = gsize * (hq / hkv);
  const int64_t items = (batch / gsize) * hkv * ((rows + 127) / 128);
  const int64_t nkt = (lp + 127) / 128;
  if (items <= 0 || nkt <= 0) return 1;
  int64_t want = (sm_count() + items - 1) / items;
  if (want > nkt) want = nkt;
  if (want < 1) want = 1;
  const int64_t per = (nkt + want - 1) / want;
  return static_cast<int>((nkt + per - 1) / per);
}

int launch_shared_prefix(const SharedPrefixLaunch& l, cudaStream_t stream) {
  const int group = l.hq / l.hkv;
  const int64_t groups = l.batch / l.gsize;
  const int64_t rows = l.gsize * group;
  const int64_t row_tiles = (rows + 127) / 128;
  const int splits = shared_prefix_splits(l.batch, l.gsize, l.hq, l.hkv, l.lp);
  const int64_t nkt = (l.lp + 127) / 128;
  const int64_t items = groups * l.hkv * row_tiles * splits;
  if (items <= 0) return PS_OK;
  if (items > 0x7fffffffLL || rows > 0x7fffffffLL)
    return fail(PS_ERR_UNSUPPORTED, "shared-prefix problem too large");
  CUtensorMap mk, mv;
  if (!make_map_3d(&mk, l.k_pre, kHeadDim, l.lp, groups * l.hkv, 64, 128) ||
      !make_map_3d(&mv, l.v_pre, kHeadDim, l.lp, groups * l.hkv, 64, 128))
    return PS_ERR_CUDA;
  SpArgs a;
  a.q = static_cast<const __nv_bfloat16*>(l.q);
  a.pos = l.pos;
  a.o = l.o_pre;
  a.lse2 = l.lse2_pre;
  a.status = l.status;
  a.hq = l.hq;
  a.hkv = l.hkv;
  a.group = group;
  a.gsize = static_cast<int32_t>(l.gsize);
  a.lp = l.lp;
  a.nkt = (l.lp + 127) / 128;
  a.row_tiles = static_cast<int32_t>(row_tiles);
  a.splits = splits;
  a.per = static_cast<int32_t>((nkt + splits - 1) / splits);
  a.split_rows = l.batch * l.hq;
  a.scale_log2 = l.scale * kLog2e;
  static bool attr[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr[dev]) {
    const int rc = check_cuda(cudaFuncSetAttribute(shared_prefix_kernel,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   static_cast<int>(kSpSmem)),
                              "cudaFuncSetAttribute(shared_prefix_kernel)");
    if (rc != PS_OK) return rc;
    attr[dev] = true;
  }
  return check_cuda(launch_pdl(shared_prefix_kernel, dim3(static_cast<unsigned>(items)),
                               dim3(kSpThreads), kSpSmem, stream, mk, mv, a),
                    "shared_prefix_kernel launch");
}

}  // namespace ps
