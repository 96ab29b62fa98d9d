// Masked prefill backward (dQ, dK, dV) on 5th-generation tensor cores, sm_100a.
//
// What it computes ("Prefix Sliding 完全拆解", §截断回传: the trainer back-propagates through
// the masked attention it ran over the last 4W tokens): with P_ij the masked softmax of
// s_ij = scale <q_i, k_j> over j in V(i) (eq. A(i), §核心机制), and D_i = <dO_i, O_i>,
//   dV_j = sum_i P_ij dO_i,   dS_ij = P_ij (<dO_i, V_j> - D_i),
//   dQ_i = scale sum_j dS_ij K_j,   dK_j = scale sum_i dS_ij Q_i,
// dK and dV summed over the query heads of a KV head.  P is rebuilt from the forward's
// log-sum-exp, so no running max is needed.  Only the tiles of the two-level plan
// (§Kernel 实现) are visited; PARTIAL tiles are masked element-wise.
//
// Three kernels:
//   bwd_prep_kernel - -D_i and -lse_i*log2(e) per (batch, head, row) into workspace rows
//             padded to whole 128-row tiles (padding: 0 and -inf, so padded rows contribute
//             nothing); zeroes the key-tile work counter.
//   bwd_dkdv_kernel - key-tile-major over (batch, KV head, key tile) items taken from an
//             atomic counter (a prefix key tile is seen by every later query tile, a window
//             key tile by about W/128 of them, so static striding would leave SMs idle): per
//             (query head of the group, query tile), S^T = K Q^T and dP^T = V dO^T into
//             TMEM, P^T and dS^T as bf16 in the columns that held S^T (two score buffers
//             swap roles every pair), dV += P^T dO and dK += dS^T Q in TMEM
//             across the whole group, so no atomics are needed.  It also stores each dS^T
//             tile (bf16) for the dQ pass.
//   bwd_dq_kernel - dQ = scale * dS K over the plan: a GEMM reading the stored dS^T tiles as
//             the MN-major A operand, so S and dP are formed only once.
// Both big kernels use the forward's roles: warps 0-7 two softmax warpgroups (group g owns
// columns [64g, 64g+64) of every TMEM lane), warps 8-9 TMA producers, warp 10 issues the
// smem x smem products (and owns TMEM), warp 11 the TMEM x smem accumulations.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "ps_device.cuh"
#include "ps_internal.h"
#include "ps_ranges.cuh"

namespace ps {
namespace {

constexpr int kT = 128;  // query and key tile rows
static_assert(kPrefillBq == kT && kPrefillBk == kT, "backward assumes square 128-row tiles");
constexpr int kBoxBytes = 128 * 128;       // [128 rows][64 bf16], 128-byte swizzle
constexpr int kTileBytes = 2 * kBoxBytes;  // [128 rows][128 bf16]
constexpr int kGroups = 2;
constexpr int kCols = 64;  // columns per softmax group
constexpr int kSoftmaxWarps = 8;
constexpr int kProdA = 8;
constexpr int kProdB = 9;
constexpr int kIssA = 10;
constexpr int kIssB = 11;
constexpr int kThreads = 12 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kPrepThreads = 256;
constexpr int kItemRing = 4;

struct BwdArgs {
  int32_t* status;
  int64_t seq, s_pad;
  int32_t batch, hq, hkv, group, nq;
  int32_t lp, w;
  float scale, scale_log2;
  const float* nl;  // [B][Hq][s_pad]: -lse * log2(e)
  const float* nd;  // [B][Hq][s_pad]: -D
  const int32_t* off;  // query-tile-major plan: [nq + 1] offsets
  const int32_t* ent;  // [n][2] (k_tile, flag)
  int32_t* counter;    // key-tile work counter
  __nv_bfloat16* ds;   // dS^T tiles [B * Hq * n_plan][16 query chunks][128 key rows][8]
  int64_t n_plan;      // plan entries per (batch, head)
  __nv_bfloat16* dq;   // [B, S, Hq, D]
  __nv_bfloat16* dk;   // [B, S, Hkv, D]
  __nv_bfloat16* dv;
};

// Bulk copy global -> shared with an L2 cache-policy hint.
__device__ __forceinline__ void bulk_load_hint(void* smem_dst, const void* gsrc, uint32_t bytes,
                                               uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 16-byte global store with the streaming (evict-first) cache operator: data written once
// and read back much later by another kernel.
__device__ __forceinline__ void st_global_cs(void* gdst, uint4 v) {
  asm volatile("st.global.cs.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(gdst), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// K-major 128x128 x 128x128 product: both operands [128 rows][128 cols] in two 64-column
// 128-byte-swizzled halves; 16 columns = 32 B per step inside a half.
__device__ __forceinline__ void mma_kmajor(uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr) {
  constexpr uint32_t idesc = umma_idesc_bf16(128, 128, false);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
    umma_ss(d_tmem, umma_desc_sw128(a_addr + off, 16, 1024),
            umma_desc_sw128(b_addr + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

// D += A * B[rows 64 grp .. 64 grp + 63] for one softmax group: A = the group's bf16 pairs in
// TMEM (32 columns from a_buf + 64 grp, 8 columns per 16 rows of B), B = smem [128 rows][128
// cols] MN-major.
__device__ __forceinline__ void mma_tmem_a(uint32_t d_tmem, uint32_t a_buf, uint32_t b_addr,
                                           int grp, bool first) {
  constexpr uint32_t idesc = umma_idesc_bf16(128, 128, true);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int kk = 4 * grp + i;
    // B rows 16kk..16kk+15: 2048 B per step; 64-column halves 16 KB apart (LBO), 8-row
    // groups 1024 B apart (SBO)
    const uint64_t bdesc = umma_desc_sw128(b_addr + kk * 2048, kBoxBytes, 1024);
    umma_ts(d_tmem, a_buf + 64 * grp + 8 * i, bdesc, idesc, (first && i == 0) ? 0u : 1u);
  }
}

// The half `hf` (B rows 64 grp + 32 hf .. + 31, A columns 64 grp + 16 hf .. + 15) of
// mma_tmem_a.
__device__ __forceinline__ void mma_tmem_a_half(uint32_t d_tmem, uint32_t a_buf, uint32_t b_addr,
                                                int grp, int hf, bool first) {
  constexpr uint32_t idesc = umma_idesc_bf16(128, 128, true);
#pragma unroll
  for (int i = 2 * hf; i < 2 * hf + 2; ++i) {
    const int kk = 4 * grp + i;
    const uint64_t bdesc = umma_desc_sw128(b_addr + kk * 2048, kBoxBytes, 1024);
    umma_ts(d_tmem, a_buf + 64 * grp + 8 * i, bdesc, idesc, (first && i == 0) ? 0u : 1u);
  }
}

__device__ __forceinline__ void load64(uint32_t taddr, float (&x)[kCols]) {
  uint32_t raw[2][32];
  tmem_ld32(taddr, raw[0]);
  tmem_ld32(taddr + 32, raw[1]);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int i = 0; i < 32; ++i) x[32 * c + i] = __uint_as_float(raw[c][i]);
}

// Bit c (c < 64) set iff c + base lies in [lo, hi).
__device__ __forceinline__ uint64_t span_bits(int64_t lo, int64_t hi, int64_t base) {
  lo -= base;
  hi -= base;
  if (lo < 0) lo = 0;
  if (hi > 64) hi = 64;
  if (hi <= lo) return 0ull;
  const uint64_t len = static_cast<uint64_t>(hi - lo);
  return (len >= 64 ? ~0ull : ((1ull << len) - 1ull)) << lo;
}

// ------------------------------------------------------------------ prep
// Rows are taken in memory order (batch, row, head): 16 lanes read one 256-byte row of O
// and of dO with 16-byte loads, so a warp covers two rows per step.  Padded rows (past seq)
// get -D = 0 and -lse*log2(e) = -inf.
__global__ void __launch_bounds__(kPrepThreads)
    bwd_prep_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
                    const float* __restrict__ lse, int64_t seq, int32_t hq, int64_t s_pad,
                    int64_t batch, float* __restrict__ nl, float* __restrict__ nd,
                    int32_t* __restrict__ counter) {
  pdl_trigger();
  pdl_wait();
  const int64_t tid = (int64_t)blockIdx.x * kPrepThreads + threadIdx.x;
  if (tid == 0) *counter = 0;
  const int64_t real = batch * seq * hq;   // rows with data, (b, i, h) order
  const int64_t half_warps = (int64_t)gridDim.x * kPrepThreads / 16;
  const int sub = threadIdx.x & 15;
  for (int64_t row = tid >> 4; row < real; row += half_warps) {
    const uint4 o = reinterpret_cast<const uint4*>(out + row * kHeadDim)[sub];
    const uint4 d = reinterpret_cast<const uint4*>(dout + row * kHeadDim)[sub];
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&d);
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(o2[e]), y = __bfloat1622float2(d2[e]);
      dot = fmaf(x.x, y.x, fmaf(x.y, y.y, dot));
    }
#pragma unroll
    for (int sh = 8; sh > 0; sh >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, sh);
    if (sub == 0) {
      const int64_t h = row % hq, bi = row / hq;
      const int64_t i = bi % seq, b = bi / seq;
      const int64_t srow = (b * hq + h) * s_pad + i;
      nd[srow] = -dot;
      nl[srow] = -lse[(b * hq + h) * seq + i] * kLog2e;
    }
  }
  // padding rows [seq, s_pad) of every (batch, head)
  const int64_t pad = s_pad - seq;
  for (int64_t k = tid; k < batch * hq * pad; k += (int64_t)gridDim.x * kPrepThreads) {
    const int64_t bh = k / pad, i = seq + k % pad;
    nd[bh * s_pad + i] = 0.f;
    nl[bh * s_pad + i] = -INFINITY;
  }
}

// ------------------------------------------------------------------ dQ
// dQ_i = scale * sum over the planned key tiles of dS K, with dS stored by the key-tile kernel
// (bf16 dS^T tiles, [key row][query col]): a plain GEMM over the plan, read as the MN-major A
// operand.  Persistent over (batch, head, query tile) items, heaviest first; warp 4 streams
// (dS tile, K tile) pairs through a 3-stage ring, warp 5 issues dQ[buf] += dS K into one of two
// TMEM accumulators, warps 0-3 drain the finished accumulator (scale, bf16, one row each) while
// the next item accumulates in the other.
constexpr int kDqThreads = 192;
constexpr int kDqStages = 3;
constexpr size_t kDqSmem = 1024 + size_t(kDqStages) * 2 * kTileBytes + 256;

__global__ void __launch_bounds__(kDqThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap mk, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sDS = smem;                              // [kDqStages] dS tiles (no swizzle)
  uint8_t* sK = sDS + kDqStages * kTileBytes;       // [kDqStages] K tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sK + kDqStages * kTileBytes);
  uint64_t* full = bars;                        // [kDqStages]
  uint64_t* empty = bars + kDqStages;           // [kDqStages]
  uint64_t* acc_full = bars + 2 * kDqStages;    // [2]
  uint64_t* acc_free = acc_full + 2;            // [2]
  uint64_t* mma_done = acc_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int64_t bh = (int64_t)a.batch * a.hq;
  const int64_t n_items = bh * a.nq;
  auto item_of = [&](int64_t it, int& qt, int& b, int& head) {
    qt = a.nq - 1 - static_cast<int>(it / bh);  // heaviest query tiles first
    const int rem = static_cast<int>(it % bh);
    head = rem % a.hq;
    b = rem / a.hq;
  };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDqStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_free[s], 4);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) prefetch_tensormap(&mk);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // the dS tiles come from the key-tile kernel launched just before

  if (warp == 4) {
    if (lane == 0) {
      int64_t g = 0;
      bool alive = true;
      for (int64_t it = blockIdx.x; alive && it < n_items; it += gridDim.x) {
        int qt, b, head;
        item_of(it, qt, b, head);
        const int kvh = head / a.group;
        const int e0 = a.off[qt];
        const int n = a.off[qt + 1] - e0;
        const int64_t tile0 = ((int64_t)b * a.hq + head) * a.n_plan + e0;
        for (int j = 0; j < n; ++j, ++g) {
          const int s = static_cast<int>(g % kDqStages);
          if (g >= kDqStages &&
              !mbar_wait(&empty[s], static_cast<uint32_t>(((g / kDqStages) - 1) & 1), a.status)) {
            alive = false;
            break;
          }
          const int kt = a.ent[2 * (e0 + j)];
          mbar_arrive_expect_tx(&full[s], 2 * kTileBytes);
          uint8_t* ds = sDS + s * kTileBytes;
          uint8_t* k = sK + s * kTileBytes;
          // each stored tile is read once: keep it from displacing the K tiles in L2
          bulk_load_hint(ds, a.ds + (tile0 + j) * kT * kT, kTileBytes, &full[s],
                         l2_policy_evict_first());
          tma_load_4d(k, &mk, 0, kvh, kt * kT, b, &full[s]);
          tma_load_4d(k + kBoxBytes, &mk, 64, kvh, kt * kT, b, &full[s]);
        }
      }
      for (int64_t j = (g > kDqStages ? g - kDqStages : 0); j < g; ++j)
        mbar_wait(&full[j % kDqStages], static_cast<uint32_t>((j / kDqStages) & 1), a.status);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // A = dS [128 query rows][128 keys], MN-major without swizzle: the stored tile is
      // [query chunk][key row][8 bf16], i.e. core matrices of 8 queries x 8 keys (128 B),
      // 2048 B apart along the queries (SBO) and 128 B apart along the keys (LBO); a 16-key
      // step advances 256 B.  B = K [128 keys][128 dims], MN-major, 128-byte swizzle: 2048 B
      // per 16-key step, 64-column halves 16 KB apart (LBO), 8-row groups 1024 B (SBO).
      constexpr uint32_t idesc = umma_idesc_bf16(128, 128, true, true);
      const uint32_t ds_addr = smem_u32(sDS), k_addr = smem_u32(sK);
      int64_t g = 0;
      int li = 0;
      bool ok = true;
      for (int64_t it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++li) {
        int qt, b, head;
        item_of(it, qt, b, head);
        const int n = a.off[qt + 1] - a.off[qt];
        const int ab = li & 1;
        if (li >= 2 &&
            !mbar_wait(&acc_free[ab], static_cast<uint32_t>(((li >> 1) - 1) & 1), a.status)) {
          ok = false;
          break;
        }
        for (int j = 0; j < n; ++j, ++g) {
          const int s = static_cast<int>(g % kDqStages);
          if (!mbar_wait(&full[s], static_cast<uint32_t>((g / kDqStages) & 1), a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t da = ds_addr + s * kTileBytes, kb = k_addr + s * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            umma_ss(tmem + 128u * ab, umma_desc_noswz(da + kk * 256, 128, 2048),
                    umma_desc_sw128(kb + kk * 2048, kBoxBytes, 1024), idesc,
                    (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, a.status);
    }
  } else {
    // epilogue warps: row r of the finished accumulator -> dQ (times the softmax scale)
    const int r = threadIdx.x;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    int li = 0;
    bool ok = true;
    for (int64_t it = blockIdx.x; it < n_items; it += gridDim.x, ++li) {
      int qt, b, head;
      item_of(it, qt, b, head);
      const int ab = li & 1;
      ok = ok && __all_sync(0xffffffffu, mbar_wait(&acc_full[ab],
                                                   static_cast<uint32_t>((li >> 1) & 1),
                                                   a.status));
      if (!ok) break;
      tc_fence_after();
      const int64_t row = (int64_t)qt * kT + r;
      __nv_bfloat16* dst = a.dq + (((int64_t)b * a.seq + row) * a.hq + head) * kHeadDim;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t raw[32];
        tmem_ld32(lane_base + 128u * ab + 32 * c, raw);
        tmem_wait_ld();
        if (c == 3) {
          // the accumulator is in registers: the item after next may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_free[ab]);
        }
        if (row < a.seq) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            d4[v] = make_uint4(
                cvt_bf16x2(a.scale * __uint_as_float(raw[8 * v]), a.scale * __uint_as_float(raw[8 * v + 1])),
                cvt_bf16x2(a.scale * __uint_as_float(raw[8 * v + 2]), a.scale * __uint_as_float(raw[8 * v + 3])),
                cvt_bf16x2(a.scale * __uint_as_float(raw[8 * v + 4]), a.scale * __uint_as_float(raw[8 * v + 5])),
                cvt_bf16x2(a.scale * __uint_as_float(raw[8 * v + 6]), a.scale * __uint_as_float(raw[8 * v + 7])));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------ dK, dV
// TMEM: two 128-column score buffers T0 [0,128) and T1 [128,256), dV [256,384), dK
// [384,512).  Pair g forms S^T in T[g & 1] and dP^T in T[(g + 1) & 1].  The softmax warps
// load S^T, write P^T (bf16) over the first 32 of their group's 64 columns of the same buffer
// and, once they have loaded dP^T, dS^T (bf16) over the other 32; so T[(g + 1) & 1] is free
// for S^T of pair g + 1 as soon as dP^T is in registers, and T[g & 1] takes dP^T of pair
// g + 1 once the dV and dK products have read P^T and dS^T.  So the next pair's scores wait
// for this pair's dP^T to be loaded, not for its dV products.
constexpr uint32_t kKColT = 0;    // T0; T1 = kKColT + 128
constexpr uint32_t kKColDsOff = 32;  // dS^T: 32 columns after P^T in the group's slice
constexpr uint32_t kKColDV = 256;
constexpr uint32_t kKColDK = 384;
constexpr int kStatBytes = kT * 4;  // one tile of -lse*log2e (or -D)
constexpr size_t kDkdvSmem = 1024 + 6 * size_t(kTileBytes) + 4 * kStatBytes + 512;

struct KvItem {
  int b, kvh, kt;
  int qlo, nqt;
};
__device__ __forceinline__ KvItem kv_item(int64_t it, const BwdArgs& a) {
  KvItem m;
  const int64_t per = (int64_t)a.batch * a.hkv;
  m.kt = static_cast<int>(it / per);  // ascending key tiles: prefix tiles (the heaviest) first
  const int rem = static_cast<int>(it % per);
  m.kvh = rem % a.hkv;
  m.b = rem / a.hkv;
  int64_t lo = 0, hi = -1;
  ktile_qrange(m.kt, a.seq, a.lp, a.w, kT, &lo, &hi);
  m.qlo = static_cast<int>(lo);
  m.nqt = static_cast<int>(hi - lo + 1);
  return m;
}

__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mdo,
                    const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                    const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + kTileBytes;
  uint8_t* sQ = sV + kTileBytes;      // [2 stages]
  uint8_t* sDO = sQ + 2 * kTileBytes;  // [2 stages]
  float* sNL = reinterpret_cast<float*>(sDO + 2 * kTileBytes);  // [2][128]
  float* sND = sNL + 2 * kT;                                      // [2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sND + 2 * kT);
  uint64_t* item_full = bars;                  // [kItemRing]
  uint64_t* item_empty = bars + kItemRing;     // [kItemRing]
  uint64_t* kv_full = bars + 2 * kItemRing;
  uint64_t* kv_empty = kv_full + 1;
  uint64_t* st_full = kv_full + 2;   // [2]
  uint64_t* st_empty = kv_full + 4;  // [2]
  uint64_t* s_full = kv_full + 6;
  uint64_t* dp_full = kv_full + 7;
  uint64_t* p_ready = kv_full + 8;    // [2 groups][2 halves of the group's 64 query columns]
  uint64_t* ds_ready = kv_full + 12;  // [2 groups]
  uint64_t* dp_loaded = kv_full + 14;  // softmax warps: dP^T of the pair is in registers
  uint64_t* pd_free = kv_full + 15;    // the pair's dV and dK products have read P^T, dS^T
  uint64_t* acc_full = kv_full + 16;
  uint64_t* acc_free = kv_full + 17;
  uint64_t* mma_done = kv_full + 18;
  int32_t* s_items = reinterpret_cast<int32_t*>(kv_full + 19);  // [kItemRing]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_items + kItemRing);

  const int64_t n_items = (int64_t)a.batch * a.hkv * a.nq;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int kItemReaders = 3 + kSoftmaxWarps;  // producer A, both issuers, softmax warps

  if (threadIdx.x == 0) {
    for (int i = 0; i < kItemRing; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], kItemReaders);
    }
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1);
      mbar_init(&p_ready[2 * s], 4);
      mbar_init(&p_ready[2 * s + 1], 4);
      mbar_init(&ds_ready[s], 4);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(dp_loaded, kSoftmaxWarps);
    mbar_init(pd_free, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, kSoftmaxWarps);
    mbar_init(mma_done, 2);
    fence_mbar_init();
  }
  if (warp == kIssA) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProdA && lane == 0) {
    prefetch_tensormap(&mq);
    prefetch_tensormap(&mdo);
    prefetch_tensormap(&mk);
    prefetch_tensormap(&mv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // row statistics and the zeroed counter come from earlier kernels

  // Item i of this CTA from the ring (slot i % kItemRing); -1 on timeout.
  auto next_item = [&](int li) -> int64_t {
    const int slot = li % kItemRing;
    if (!mbar_wait(&item_full[slot], static_cast<uint32_t>((li / kItemRing) & 1), a.status))
      return -1;
    return *reinterpret_cast<volatile int32_t*>(&s_items[slot]);
  };

  if (warp == kProdB) {
    // ---------------------------------------------------- item fetcher + K/V producer
    if (lane == 0) {
      int li = 0;
      for (;; ++li) {
        const int slot = li % kItemRing;
        if (li >= kItemRing &&
            !mbar_wait(&item_empty[slot], static_cast<uint32_t>(((li / kItemRing) - 1) & 1),
                       a.status))
          break;
        // take the next item only once this CTA's K/V buffer is free again
        if (li > 0 && !mbar_wait(kv_empty, (li - 1) & 1, a.status)) break;
        const int32_t it = atomicAdd(a.counter, 1);
        s_items[slot] = it >= n_items ? static_cast<int32_t>(n_items) : it;
        mbar_arrive(&item_full[slot]);
        if (it >= n_items) break;
        const KvItem m = kv_item(it, a);
        mbar_arrive_expect_tx(kv_full, 2 * kTileBytes);
        tma_load_4d(sK, &mk, 0, m.kvh, m.kt * kT, m.b, kv_full);
        tma_load_4d(sK + kBoxBytes, &mk, 64, m.kvh, m.kt * kT, m.b, kv_full);
        tma_load_4d(sV, &mv, 0, m.kvh, m.kt * kT, m.b, kv_full);
        tma_load_4d(sV + kBoxBytes, &mv, 64, m.kvh, m.kt * kT, m.b, kv_full);
      }
      // li items were loaded (the last fetch returned the end marker or a wait failed)
      if (li > 0) mbar_wait(kv_full, (li - 1) & 1, a.status);
    }
  } else if (warp == kProdA) {
    // ---------------------------------------------------- Q, dO and row statistics
    if (lane == 0) {
      int64_t g = 0;
      bool alive = true;
      for (int li = 0; alive; ++li) {
        const int64_t it = next_item(li);
        if (it < 0) break;
        mbar_arrive(&item_empty[li % kItemRing]);
        if (it >= n_items) break;
        const KvItem m = kv_item(it, a);
        const int n = a.group * m.nqt;
        for (int j = 0; j < n; ++j, ++g) {
          const int st = static_cast<int>(g & 1);
          if (g >= 2 &&
              !mbar_wait(&st_empty[st], static_cast<uint32_t>(((g >> 1) - 1) & 1), a.status)) {
            alive = false;
            break;
          }
          const int h = m.kvh * a.group + j / m.nqt;
          const int qt = m.qlo + j % m.nqt;
          mbar_arrive_expect_tx(&st_full[st], 2 * kTileBytes + 2 * kStatBytes);
          uint8_t* q = sQ + st * kTileBytes;
          uint8_t* d = sDO + st * kTileBytes;
          tma_load_4d(q, &mq, 0, h, qt * kT, m.b, &st_full[st]);
          tma_load_4d(q + kBoxBytes, &mq, 64, h, qt * kT, m.b, &st_full[st]);
          tma_load_4d(d, &mdo, 0, h, qt * kT, m.b, &st_full[st]);
          tma_load_4d(d + kBoxBytes, &mdo, 64, h, qt * kT, m.b, &st_full[st]);
          const int64_t srow = ((int64_t)m.b * a.hq + h) * a.s_pad + (int64_t)qt * kT;
          bulk_load(sNL + st * kT, a.nl + srow, kStatBytes, &st_full[st]);
          bulk_load(sND + st * kT, a.nd + srow, kStatBytes, &st_full[st]);
        }
      }
      for (int64_t j = (g > 2 ? g - 2 : 0); j < g; ++j)
        mbar_wait(&st_full[j & 1], static_cast<uint32_t>((j >> 1) & 1), a.status);
    }
  } else if (warp == kIssA) {
    // ---------------------------------------------------- S^T = K Q^T, dP^T = V dO^T
    if (lane == 0) {
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      const uint32_t q_addr = smem_u32(sQ), do_addr = smem_u32(sDO);
      int64_t g = 0;
      bool ok = true;
      for (int li = 0; ok; ++li) {
        const int64_t it = next_item(li);
        if (it < 0) break;
        mbar_arrive(&item_empty[li % kItemRing]);
        if (it >= n_items) break;
        const KvItem m = kv_item(it, a);
        const int n = a.group * m.nqt;
        if (!mbar_wait(kv_full, li & 1, a.status)) break;
        for (int j = 0; j < n; ++j, ++g) {
          const int st = static_cast<int>(g & 1);
          const uint32_t prev = static_cast<uint32_t>((g - 1) & 1);
          if (!mbar_wait(&st_full[st], static_cast<uint32_t>((g >> 1) & 1), a.status) ||
              (g >= 1 && !mbar_wait(dp_loaded, prev, a.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          // S^T into T[g & 1], which held dP^T of pair g - 1
          mma_kmajor(tmem + kKColT + 128 * st, k_addr, q_addr + st * kTileBytes);
          umma_commit(s_full);
          if (g >= 1 && !mbar_wait(pd_free, prev, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // dP^T into T[(g + 1) & 1], which held P^T and dS^T of pair g - 1
          mma_kmajor(tmem + kKColT + 128 * (st ^ 1), v_addr, do_addr + st * kTileBytes);
          umma_commit(dp_full);
        }
        if (!ok) break;
        umma_commit(kv_empty);  // K and V of this item are no longer read
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, a.status);
    }
  } else if (warp == kIssB) {
    // ---------------------------------------------------- dV += P^T dO, dK += dS^T Q
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ), do_addr = smem_u32(sDO);
      int64_t g = 0;
      bool ok = true;
      for (int li = 0; ok; ++li) {
        const int64_t it = next_item(li);
        if (it < 0) break;
        mbar_arrive(&item_empty[li % kItemRing]);
        if (it >= n_items) break;
        const KvItem m = kv_item(it, a);
        const int n = a.group * m.nqt;
        for (int j = 0; j < n; ++j, ++g) {
          const int st = static_cast<int>(g & 1);
          const uint32_t ph = static_cast<uint32_t>(g & 1);
          if (j == 0 && li > 0 && !mbar_wait(acc_free, (li - 1) & 1, a.status)) {
            ok = false;
            break;
          }
          // each group publishes its P in two halves of 32 query columns: the dV products of
          // a half go out as soon as it is in
#pragma unroll
          for (int gr = 0; gr < kGroups; ++gr) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              if (!mbar_wait(&p_ready[2 * gr + hf], ph, a.status)) {
                ok = false;
                break;
              }
              tc_fence_after();
              mma_tmem_a_half(tmem + kKColDV, tmem + kKColT + 128 * st,
                              do_addr + st * kTileBytes, gr, hf, j == 0 && gr == 0);
            }
            if (!ok) break;
          }
          if (!ok) break;
#pragma unroll
          for (int gr = 0; gr < kGroups; ++gr) {
            if (!mbar_wait(&ds_ready[gr], ph, a.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            mma_tmem_a(tmem + kKColDK, tmem + kKColT + 128 * st + kKColDsOff,
                       q_addr + st * kTileBytes, gr,
                       j == 0 && gr == 0);
          }
          if (!ok) break;
          umma_commit(pd_free);
          umma_commit(&st_empty[st]);
        }
        if (!ok) break;
        umma_commit(acc_full);
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, a.status);
    }
  } else {
    // ---------------------------------------------------- softmax warpgroups
    // TMEM lane r = key row kt*128 + r; group wg owns query columns [64 wg, 64 wg + 64).
    const int wg = threadIdx.x >> 7;
    const int r = threadIdx.x & 127;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t cs0 = static_cast<uint32_t>(kCols * wg);
    const uint64_t sl2x2 = pack_f32x2(a.scale_log2, a.scale_log2);
    bool ok = true;
    int64_t g = 0;
    for (int li = 0;; ++li) {
      const int64_t it = next_item(li);
      __syncwarp();
      if (lane == 0 && it >= 0) mbar_arrive(&item_empty[li % kItemRing]);
      if (it < 0 || it >= n_items) break;
      const KvItem m = kv_item(it, a);
      const int n = a.group * m.nqt;
      const int64_t kr = (int64_t)m.kt * kT + r;  // this thread's key
      // queries that see key kr: [kr, vis_end)
      int64_t vis_end = kr;
      if (kr < a.seq) vis_end = (kr < a.lp || kr + a.w > a.seq) ? a.seq : kr + a.w;
      for (int j = 0; j < n; ++j, ++g) {
        const int st = static_cast<int>(g & 1);
        const uint32_t ph = static_cast<uint32_t>(g & 1);
        const int qt = m.qlo + j % m.nqt;
        const int flag = classify_tile(qt, m.kt, a.seq, a.lp, a.w, kT, kT);
        // this (query tile, key tile)'s dS^T tile in the store: query tile qt's plan offset
        // plus the key tile's closed-form position in it, formed before the scores are
        // waited for
        __nv_bfloat16* ds_row;
        {
          const int64_t e = a.off[qt] + plan_index(qt, m.kt, a.lp, a.w, kT);
          const int h = m.kvh * a.group + j / m.nqt;
          // tile layout: [16 column chunks of 8 query cols][128 key rows][8 bf16], so the
          // 32 rows of a warp store 512 contiguous bytes per chunk
          ds_row = a.ds + (((int64_t)m.b * a.hq + h) * a.n_plan + e) * kT * kT + r * 8;
        }
        ok = ok && __all_sync(0xffffffffu,
                              mbar_wait(s_full, ph, a.status) &&
                                  mbar_wait(&st_full[st], static_cast<uint32_t>((g >> 1) & 1),
                                            a.status));
        if (!ok) continue;
        tc_fence_after();
        float x[kCols];
        const uint32_t t_s = lane_base + kKColT + 128 * st;         // S^T, then P^T, dS^T
        const uint32_t t_dp = lane_base + kKColT + 128 * (st ^ 1);  // dP^T
        load64(t_s + cs0, x);
        if (flag == PS_TILE_PARTIAL) {
          const uint64_t vis = span_bits(kr, vis_end, (int64_t)qt * kT + cs0);
#pragma unroll
          for (int i = 0; i < kCols; ++i)
            if (!((vis >> i) & 1ull)) x[i] = -INFINITY;
        }
        const float4* nl = reinterpret_cast<const float4*>(sNL + st * kT + cs0);
        const float4* nd4 = reinterpret_cast<const float4*>(sND + st * kT + cs0);
        // P over this group's own columns, published in two halves of 32 query columns so
        // that the first half's dV products overlap the second half's exponentials
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[kCols / 4];
#pragma unroll
          for (int ii = 0; ii < kCols / 8; ++ii) {
            const int i = hf * (kCols / 8) + ii;
            const float4 l = nl[i];
            const float2 e0 = unpack_f32x2(
                ffma2(pack_f32x2(x[4 * i], x[4 * i + 1]), sl2x2, pack_f32x2(l.x, l.y)));
            const float2 e1 = unpack_f32x2(
                ffma2(pack_f32x2(x[4 * i + 2], x[4 * i + 3]), sl2x2, pack_f32x2(l.z, l.w)));
            x[4 * i] = fast_exp2(e0.x);
            x[4 * i + 1] = fast_exp2(e0.y);
            x[4 * i + 2] = fast_exp2(e1.x);
            x[4 * i + 3] = fast_exp2(e1.y);
            pk[2 * ii] = cvt_bf16x2(x[4 * i], x[4 * i + 1]);
            pk[2 * ii + 1] = cvt_bf16x2(x[4 * i + 2], x[4 * i + 3]);
          }
          tmem_st16(t_s + cs0 + 16 * hf, pk);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_ready[2 * wg + hf]);
        }
        ok = ok && __all_sync(0xffffffffu, mbar_wait(dp_full, ph, a.status));
        if (!ok) continue;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t raw[32];
          tmem_ld32(t_dp + cs0 + 32 * c, raw);
          tmem_wait_ld();
          if (c == 1) {
            // dP^T is in registers: its buffer can take the next pair's S^T
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dp_loaded);
          }
          uint32_t dk[16];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int e = 32 * c + 4 * i;
            const float4 d = nd4[e / 4];
            const float2 v0 = unpack_f32x2(
                fmul2(pack_f32x2(x[e], x[e + 1]),
                      fadd2(pack_f32x2(__uint_as_float(raw[4 * i]), __uint_as_float(raw[4 * i + 1])),
                            pack_f32x2(d.x, d.y))));
            const float2 v1 = unpack_f32x2(
                fmul2(pack_f32x2(x[e + 2], x[e + 3]),
                      fadd2(pack_f32x2(__uint_as_float(raw[4 * i + 2]),
                                       __uint_as_float(raw[4 * i + 3])),
                            pack_f32x2(d.z, d.w))));
            dk[2 * i] = cvt_bf16x2(v0.x, v0.y);
            dk[2 * i + 1] = cvt_bf16x2(v1.x, v1.y);
          }
          tmem_st16(t_s + cs0 + kKColDsOff + 16 * c, dk);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int chunk = (cs0 >> 3) + 4 * c + v;  // query cols [8 chunk, 8 chunk + 8)
            st_global_cs(ds_row + chunk * kT * 8,
                         make_uint4(dk[4 * v], dk[4 * v + 1], dk[4 * v + 2], dk[4 * v + 3]));
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ds_ready[wg]);
      }
      // epilogue: dV and dK (times the softmax scale) of this key tile
      const bool fin = __all_sync(0xffffffffu, ok && mbar_wait(acc_full, li & 1, a.status));
      ok = ok && fin;
      if (!fin) continue;
      tc_fence_after();
      uint32_t pv[kCols / 2], pkk[kCols / 2];
      {
        float acc[kCols];
        load64(lane_base + kKColDV + cs0, acc);
#pragma unroll
        for (int i = 0; i < kCols / 2; ++i) pv[i] = cvt_bf16x2(acc[2 * i], acc[2 * i + 1]);
        load64(lane_base + kKColDK + cs0, acc);
#pragma unroll
        for (int i = 0; i < kCols / 2; ++i)
          pkk[i] = cvt_bf16x2(a.scale * acc[2 * i], a.scale * acc[2 * i + 1]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_free);
      if (kr < a.seq) {
        const int64_t o = (((int64_t)m.b * a.seq + kr) * a.hkv + m.kvh) * kHeadDim + cs0;
        uint4* dv = reinterpret_cast<uint4*>(a.dv + o);
        uint4* dk = reinterpret_cast<uint4*>(a.dk + o);
#pragma unroll
        for (int v = 0; v < kCols / 8; ++v) {
          dv[v] = make_uint4(pv[4 * v], pv[4 * v + 1], pv[4 * v + 2], pv[4 * v + 3]);
          dk[v] = make_uint4(pkk[4 * v], pkk[4 * v + 1], pkk[4 * v + 2], pkk[4 * v + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kIssA) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace: [plan][-lse*log2e rows][-D rows][counter][dS^T tiles of every planned tile,
// 32 KB each], for `batch` sequences per pass.
struct BwdLayout {
  size_t plan, stats, counter, ds, total;
  int64_t n_plan;
};
BwdLayout bwd_layout(int64_t batch, int32_t hq, int64_t seq, int32_t lp, int32_t w) {
  BwdLayout L;
  L.n_plan = prefill_plan_tiles(seq, lp, w);
  L.plan = prefill_plan_bytes(seq, L.n_plan);
  const int64_t s_pad = (seq + kT - 1) / kT * kT;
  L.stats = align256(size_t(batch) * hq * s_pad * 4);
  L.counter = 256;
  L.ds = size_t(batch) * hq * L.n_plan * kT * kT * 2;
  L.total = align256(L.plan) + 2 * L.stats + L.counter + L.ds;
  return L;
}

// The dS^T store of one pass is kept under this many bytes: a batch whose store would be
// larger runs in passes of fewer sequences (the workspace stops growing with the batch).
constexpr size_t kDsPassBytes = size_t(4) << 30;

// Sequences per pass: the most (up to `batch`) whose layout fits `ws_bytes`; 0 if not even
// one does.
int64_t bwd_pass_batch(int64_t batch, int32_t hq, int64_t seq, int32_t lp, int32_t w,
                       size_t ws_bytes) {
  const BwdLayout one = bwd_layout(1, hq, seq, lp, w);
  if (one.total > ws_bytes) return 0;
  int64_t lo = 1, hi = batch;  // largest n in [1, batch] with layout(n) <= ws_bytes
  while (lo < hi) {
    const int64_t mid = lo + (hi - lo + 1) / 2;
    if (bwd_layout(mid, hq, seq, lp, w).total <= ws_bytes) lo = mid; else hi = mid - 1;
  }
  return lo;
}

bool set_smem(const void* fn, size_t bytes, bool* done, const char* what, int* rc) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!done[dev]) {
    *rc = check_cuda(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(bytes)),
                     what);
    if (*rc != PS_OK) return false;
    done[dev] = true;
  }
  return true;
}

}  // namespace

size_t prefill_bwd_workspace_bytes(int64_t batch, int32_t hq, int64_t seq, int32_t lp, int32_t w) {
  const BwdLayout one = bwd_layout(1, hq, seq, lp, w);
  int64_t n = batch < 1 ? 1 : batch;
  const int64_t per_pass = static_cast<int64_t>(kDsPassBytes / (one.ds > 0 ? one.ds : 1));
  if (n > per_pass) n = per_pass < 1 ? 1 : per_pass;
  return bwd_layout(n, hq, seq, lp, w).total;
}

size_t prefill_bwd_min_workspace_bytes(int32_t hq, int64_t seq, int32_t lp, int32_t w) {
  return bwd_layout(1, hq, seq, lp, w).total;
}

namespace {

// One pass over sequences [b0, b0 + nb) of the batch (the plan is already in the workspace).
int launch_bwd_pass(const PrefillBwdLaunch& l, int64_t b0, int64_t nb, cudaStream_t stream) {
  const int64_t nq = (l.seq + kT - 1) / kT;
  const int64_t s_pad = nq * kT;
  const BwdLayout L = bwd_layout(nb, l.hq, l.seq, l.lp, l.w);
  char* ws = static_cast<char*>(l.workspace);
  const size_t qrow = size_t(l.seq) * l.hq * kHeadDim * 2;   // bytes per sequence, q-shaped
  const size_t krow = size_t(l.seq) * l.hkv * kHeadDim * 2;  // k-shaped
  const char* q = static_cast<const char*>(l.q) + b0 * qrow;
  const char* k = static_cast<const char*>(l.k) + b0 * krow;
  const char* v = static_cast<const char*>(l.v) + b0 * krow;
  const char* out = static_cast<const char*>(l.out) + b0 * qrow;
  const char* dout = static_cast<const char*>(l.dout) + b0 * qrow;
  const float* lse = l.lse + b0 * l.hq * l.seq;
  int rc = PS_OK;

  BwdArgs a;
  a.status = l.status;
  a.seq = l.seq;
  a.s_pad = s_pad;
  a.batch = static_cast<int32_t>(nb);
  a.hq = l.hq;
  a.hkv = l.hkv;
  a.group = l.hq / l.hkv;
  a.nq = static_cast<int32_t>(nq);
  a.lp = l.lp;
  a.w = l.w;
  a.scale = l.scale;
  a.scale_log2 = l.scale * kLog2e;
  a.off = reinterpret_cast<const int32_t*>(ws);
  a.ent = reinterpret_cast<const int32_t*>(ws + align256(size_t(nq + 1) * 4));
  float* nl = reinterpret_cast<float*>(ws + align256(L.plan));
  float* nd = reinterpret_cast<float*>(ws + align256(L.plan) + L.stats);
  a.nl = nl;
  a.nd = nd;
  a.counter = reinterpret_cast<int32_t*>(ws + align256(L.plan) + 2 * L.stats);
  a.ds = reinterpret_cast<__nv_bfloat16*>(ws + align256(L.plan) + 2 * L.stats + L.counter);
  a.n_plan = L.n_plan;
  a.dq = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(l.dq) + b0 * qrow);
  a.dk = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(l.dk) + b0 * krow);
  a.dv = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(l.dv) + b0 * krow);

  // row statistics: a grid of a few waves of the SMs, each half-warp striding over rows
  const int64_t sms = sm_count();
  const int64_t real_rows = nb * l.seq * l.hq;
  int64_t prep_blocks = (real_rows * 16 + kPrepThreads - 1) / kPrepThreads;
  if (prep_blocks > sms * 16) prep_blocks = sms * 16;
  if (prep_blocks < 1) prep_blocks = 1;
  rc = check_cuda(launch_pdl(bwd_prep_kernel, dim3(static_cast<unsigned>(prep_blocks)),
                             dim3(kPrepThreads), 0, stream,
                             reinterpret_cast<const __nv_bfloat16*>(out),
                             reinterpret_cast<const __nv_bfloat16*>(dout), lse, l.seq, l.hq, s_pad,
                             nb, nl, nd, a.counter),
                  "bwd_prep_kernel launch");
  if (rc != PS_OK) return rc;

  CUtensorMap mq, mdo, mk, mv;
  const uint64_t dq_dims[4] = {kHeadDim, (uint64_t)l.hq, (uint64_t)l.seq, (uint64_t)nb};
  const uint64_t dk_dims[4] = {kHeadDim, (uint64_t)l.hkv, (uint64_t)l.seq, (uint64_t)nb};
  const uint32_t box[4] = {64, 1, 128, 1};
  if (!make_map_4d(&mq, q, dq_dims, box) || !make_map_4d(&mdo, dout, dq_dims, box) ||
      !make_map_4d(&mk, k, dk_dims, box) || !make_map_4d(&mv, v, dk_dims, box))
    return PS_ERR_CUDA;


  static bool dq_attr[64] = {false}, kv_attr[64] = {false};
  if (!set_smem(reinterpret_cast<const void*>(bwd_dq_kernel), kDqSmem, dq_attr,
                "cudaFuncSetAttribute(bwd_dq_kernel)", &rc) ||
      !set_smem(reinterpret_cast<const void*>(bwd_dkdv_kernel), kDkdvSmem, kv_attr,
                "cudaFuncSetAttribute(bwd_dkdv_kernel)", &rc))
    return rc;
  const int64_t q_items = nb * l.hq * nq;
  const int64_t kv_items = nb * l.hkv * nq;
  if (q_items > 0x7fffffffLL) return fail(PS_ERR_UNSUPPORTED, "prefill backward too large");
  // dK, dV (and the dS^T tiles) first, then dQ from the stored tiles
  rc = check_cuda(
      launch_pdl(bwd_dkdv_kernel, dim3(static_cast<unsigned>(kv_items < sms ? kv_items : sms)),
                 dim3(kThreads), kDkdvSmem, stream, mq, mdo, mk, mv, a),
      "bwd_dkdv_kernel launch");
  if (rc != PS_OK) return rc;
  return check_cuda(
      launch_pdl(bwd_dq_kernel, dim3(static_cast<unsigned>(q_items < sms ? q_items : sms)),
                 dim3(kDqThreads), kDqSmem, stream, mk, a),
      "bwd_dq_kernel launch");
}

}  // namespace

int launch_prefill_bwd(const PrefillBwdLaunch& l, cudaStream_t stream) {
  const int64_t nb = bwd_pass_batch(l.batch, l.hq, l.seq, l.lp, l.w, l.ws_bytes);
  if (nb < 1) return fail(PS_ERR_WORKSPACE, "prefill backward workspace too small");
  const int64_t n_tiles = prefill_plan_tiles(l.seq, l.lp, l.w);
  int rc = check_cuda(launch_plan(l.seq, l.lp, l.w, n_tiles, l.workspace, nullptr, stream),
                      "plan_kernel launch");
  // passes of nb sequences; each writes its own rows of dq, dk and dv
  for (int64_t b0 = 0; rc == PS_OK && b0 < l.batch; b0 += nb)
    rc = launch_bwd_pass(l, b0, l.batch - b0 < nb ? l.batch - b0 : nb, stream);
  return rc;
}

}  // namespace ps
