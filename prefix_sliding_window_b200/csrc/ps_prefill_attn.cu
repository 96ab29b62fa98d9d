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
// Persistent: one CTA per SM walks the (batch, query head, 128-row query tile) items
// blockIdx.x, blockIdx.x + gridDim.x, ... (heaviest query tiles first); TMEM, barriers and
// the TMA rings live across items, so the next item's Q tile and first QK^T overlap the
// previous item's tail.  12 warps:
//   warps 8, 9 - TMA producers: warp 8 loads the query tiles (two buffers) and the K tiles
//             of the plan into a 2-stage ring, warp 9 the V tiles into a 2-stage ring (4-D
//             tensor maps, 128-byte swizzle).  A query buffer is released after its item's
//             last QK^T, a K stage when its QK^T completes, a V stage when its PV completes.
//   warp 10 - allocates 512 TMEM columns; one lane issues S[buf] = Q K^T (tcgen05.mma
//             kind::f16, A and B from smem) as soon as K is in and the buffer's previous P
//             has been consumed, so the next scores are computed while softmax runs.
//   warp 11 - one lane issues O_g += P_g V_g, g = 0, 1 (A = P from TMEM, B = V from smem,
//             MN-major; P_g, V_g: keys [64g, 64g+64) of the tile) as soon as that group's P
//             and the V tile are in.  Each issuer commits its own MMAs to mbarriers.
//   warps 0-7 - softmax, two warpgroups: row r lives in TMEM lane r; group g handles the
//             64 score columns [64g, 64g+64) of every row as an independent online softmax
//             (its own max m_g, sum l_g and accumulator O_g), so the groups never wait for
//             each other inside the loop.  On PARTIAL tiles each thread masks its slice with
//             a 64-bit interval mask built once per row; it then writes P as bf16 over the
//             first half of its own columns of the same S buffer (packed fp32x2 FMA/add, one ex2 per element) and
//             signals the MMA warp.  O_g is rescaled in TMEM only when the max of some row
//             of the warp grows by more than 8 (log2 units); otherwise P stays below 2^8
//             and the stale max keeps fp32 sums exact enough.  The decision is warp-uniform
//             because tcgen05.ld/st are warp-collective.
//   Epilogue (per item): O = (2^(m_0-M) O_0 + 2^(m_1-M) O_1) / (2^(m_0-M) l_0 + 2^(m_1-M) l_1);
//             once O is in registers the warps release it (o_free) so the next item's first
//             PV may overwrite it; each group stores half of the columns as bf16, group 0
//             the lse.
// TMEM columns: S0 [0,128), S1 [128,256), O_0 [256,384), O_1 [384,512).

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
constexpr int kGroups = 2;                // softmax warpgroups, one column slice each
constexpr int kCols = 128 / kGroups;       // score columns per group
constexpr int kSoftmaxWarps = 4 * kGroups;
constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
constexpr int kKProducerWarp = kSoftmaxWarps;
constexpr int kVProducerWarp = kSoftmaxWarps + 1;
constexpr int kMmaWarp = kSoftmaxWarps + 2;   // issues QK^T, owns TMEM
constexpr int kPvWarp = kSoftmaxWarps + 3;    // issues PV
constexpr int kThreads = (kSoftmaxWarps + 4) * 32;
constexpr int kQStages = 2;
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr int kBoxBytes = 128 * 128;        // [128 rows][64 bf16]
constexpr int kTileBytes = 2 * kBoxBytes;   // [128 rows][128 bf16]
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t col_s(int s) { return s ? 128u : 0u; }
constexpr uint32_t kColO = 256;  // O_g at kColO + 128 g
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

constexpr size_t kSmemBytes =
    1024 + kTileBytes * (kQStages + kKStages + kVStages) + 256 + 2 * 2 * kGroups * 128 * 4;

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

// Bit c of the result is set iff key k0 + c (c < 64) is visible from query `row`: the keys
// row can see are [0, min(lp, row+1)) and [max(lp, row-w+1), row+1), both cut at seq.
__device__ __forceinline__ uint64_t interval_bits(int64_t lo, int64_t hi, int64_t k0) {
  lo -= k0;
  hi -= k0;
  if (lo < 0) lo = 0;
  if (hi > 64) hi = 64;
  if (hi <= lo) return 0ull;
  const uint64_t len = static_cast<uint64_t>(hi - lo);
  const uint64_t ones = len >= 64 ? ~0ull : ((1ull << len) - 1ull);
  return ones << lo;
}
__device__ __forceinline__ uint64_t visible_bits(int64_t row, int64_t k0, int64_t seq, int32_t lp,
                                                 int32_t w) {
  const int64_t end = row + 1 < seq ? row + 1 : seq;
  const int64_t pre_end = lp < end ? lp : end;
  int64_t win_lo = row - w + 1;
  if (win_lo < lp) win_lo = lp;
  return interval_bits(0, pre_end, k0) | interval_bits(win_lo, end, k0);
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                   const __grid_constant__ CUtensorMap mv, const PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                       // [kQStages] query tiles
  uint8_t* sK = sQ + kQStages * kTileBytes;  // [kKStages]
  uint8_t* sV = sK + kKStages * kTileBytes;  // [kVStages]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kVStages * kTileBytes);
  uint64_t* q_full = bars;                           // [kQStages]
  uint64_t* q_empty = q_full + kQStages;             // [kQStages]
  uint64_t* k_full = q_empty + kQStages;             // [kKStages]
  uint64_t* k_empty = k_full + kKStages;             // [kKStages]
  uint64_t* v_full = k_empty + kKStages;             // [kVStages]
  uint64_t* v_empty = v_full + kVStages;             // [kVStages]
  uint64_t* s_full = v_empty + kVStages;             // [2]
  uint64_t* p_ready = s_full + 2;                    // [2 buffers][kGroups][2 halves]
  uint64_t* pv_done = p_ready + 4 * kGroups;          // [2]: PV of tile g -> g & 1
  uint64_t* o_free = pv_done + 2;
  uint64_t* mma_done = o_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int64_t bh = (int64_t)a.batch * a.hq;
  const int64_t n_items = bh * a.nq;
  // item it (heaviest query tiles first): qt = nq-1 - it / (batch*hq), then (b, head)
  auto item_of = [&](int64_t it, int& qt, int& b, int& head) {
    qt = a.nq - 1 - static_cast<int>(it / bh);
    const int rem = static_cast<int>(it % bh);
    head = rem % a.hq;
    b = rem / a.hq;
  };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      for (int g = 0; g < kGroups; ++g) {
        mbar_init(&p_ready[(s * kGroups + g) * 2], 4);
        mbar_init(&p_ready[(s * kGroups + g) * 2 + 1], 4);
      }
    }
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(o_free, kSoftmaxWarps);
    mbar_init(mma_done, 2);  // both MMA issuers
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kKProducerWarp && lane == 0) {
    prefetch_tensormap(&mq);
    prefetch_tensormap(&mk);
    prefetch_tensormap(&mv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // the plan comes from the kernel launched just before

  if (warp == kKProducerWarp || warp == kVProducerWarp) {
    // ------------------------------------------------------------ TMA producers
    // Warp 8 streams the query tiles (double-buffered, one per item) and the K tiles, warp 9
    // the V tiles; both walk this CTA's items and their planned tiles in order.
    if (lane == 0) {
      const bool is_k = (warp == kKProducerWarp);
      const CUtensorMap* map = is_k ? &mk : &mv;
      uint8_t* ring = is_k ? sK : sV;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const int stages = is_k ? kKStages : kVStages;
      int64_t g = 0;
      int li = 0;
      int q_issued = 0;
      bool alive = true;
      for (int64_t it = blockIdx.x; alive && it < n_items; it += gridDim.x, ++li) {
        int qt, b, head;
        item_of(it, qt, b, head);
        const int kvh = head / a.group;
        const int e0 = a.off[qt];
        const int n = a.off[qt + 1] - e0;
        if (is_k) {
          const int qb = li % kQStages;
          // the buffer's previous query tile must be done with (its item's last QK^T)
          if (li >= kQStages &&
              !mbar_wait(&q_empty[qb], ((li / kQStages) - 1) & 1, a.status)) {
            alive = false;
            break;
          }
          mbar_arrive_expect_tx(&q_full[qb], kTileBytes);
          tma_load_4d(sQ + qb * kTileBytes, &mq, 0, head, qt * kBq, b, &q_full[qb]);
          tma_load_4d(sQ + qb * kTileBytes + kBoxBytes, &mq, 64, head, qt * kBq, b, &q_full[qb]);
          ++q_issued;
        }
        for (int j = 0; j < n; ++j, ++g) {
          const int s = static_cast<int>(g % stages);
          const uint32_t ph = static_cast<uint32_t>((g / stages) & 1);
          if (g >= stages && !mbar_wait(&empty[s], ph ^ 1, a.status)) {
            alive = false;
            break;
          }
          const int kt = a.ent[2 * (e0 + j)];
          uint8_t* dst = ring + s * kTileBytes;
          mbar_arrive_expect_tx(&full[s], kTileBytes);
          tma_load_4d(dst, map, 0, kvh, kt * kBk, b, &full[s]);
          tma_load_4d(dst + kBoxBytes, map, 64, kvh, kt * kBk, b, &full[s]);
        }
      }
      // every issued copy lands before the CTA may exit
      for (int64_t j = (g > stages ? g - stages : 0); j < g; ++j)
        mbar_wait(&full[j % stages], static_cast<uint32_t>((j / stages) & 1), a.status);
      if (is_k)
        for (int j = (q_issued > kQStages ? q_issued - kQStages : 0); j < q_issued; ++j)
          mbar_wait(&q_full[j % kQStages], (j / kQStages) & 1, a.status);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ QK^T issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(128, 128, false);
      const uint32_t k_addr = smem_u32(sK);
      int64_t g = 0;
      int li = 0;
      bool ok = true;
      for (int64_t it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++li) {
        int qt, b, head;
        item_of(it, qt, b, head);
        const int n = a.off[qt + 1] - a.off[qt];
        const int qb = li % kQStages;
        if (!mbar_wait(&q_full[qb], (li / kQStages) & 1, a.status)) {
          ok = false;
          break;
        }
        const uint32_t q_addr = smem_u32(sQ + qb * kTileBytes);
        for (int j = 0; j < n; ++j, ++g) {
          const int s = static_cast<int>(g & 1);
          const int ks = static_cast<int>(g % kKStages);
          if (!mbar_wait(&k_full[ks], static_cast<uint32_t>((g / kKStages) & 1), a.status)) {
            ok = false;
            break;
          }
          // S buffer s held P of tile g-2: its PV must have finished reading it
          if (g >= 2 &&
              !mbar_wait(&pv_done[s], static_cast<uint32_t>(((g >> 1) - 1) & 1), a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kb = k_addr + ks * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // A = Q, B = K: K-major, 128-byte rows, 8-row groups 1024 B apart; 16 columns =
            // 32 B per step inside a 64-column half.
            const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
            umma_ss(tmem + col_s(s), umma_desc_sw128(q_addr + off, 16, 1024),
                    umma_desc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[s]);
          umma_commit(&k_empty[ks]);
          if (j == n - 1) umma_commit(&q_empty[qb]);
        }
      }
      umma_commit(mma_done);  // arrives once this thread's MMAs have all completed
      mbar_wait(mma_done, 0, a.status);
    }
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------ PV issuer
    // Separate from the QK^T issuer, so PV of a tile goes out as soon as its P and V are in,
    // instead of queueing behind the next tile's QK^T (which waits for an older PV).
    if (lane == 0) {
      constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 128, true);
      const uint32_t v_addr = smem_u32(sV);
      int64_t g = 0;
      int li = 0;
      bool ok = true;
      for (int64_t it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++li) {
        int qt, b, head;
        item_of(it, qt, b, head);
        const int n = a.off[qt + 1] - a.off[qt];
        for (int j = 0; j < n; ++j, ++g) {
          const int s = static_cast<int>(g & 1);
          const int vs = static_cast<int>(g % kVStages);
          if (!mbar_wait(&v_full[vs], static_cast<uint32_t>((g / kVStages) & 1), a.status)) {
            ok = false;
            break;
          }
          // the first PV of an item zero-initialises O_0 / O_1, after the previous item's
          // epilogue has read them
          if (j == 0 && li > 0 && !mbar_wait(o_free, (li - 1) & 1, a.status)) {
            ok = false;
            break;
          }
          const uint32_t vb = v_addr + vs * kTileBytes;
          // group gr's keys [64gr, 64gr+64) accumulate into its own O_gr, 32 keys at a time
          // as soon as that half of its P is in
#pragma unroll
          for (int gh = 0; gh < 2 * kGroups; ++gh) {
            const int gr = gh >> 1, hf = gh & 1;
            if (!mbar_wait(&p_ready[(s * kGroups + gr) * 2 + hf],
                           static_cast<uint32_t>((g >> 1) & 1), a.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 4 * gr + 2 * hf; kk < 4 * gr + 2 * hf + 2; ++kk) {
              // B = V[16 keys][128 d]: MN-major, 64-column halves 16 KB apart (LBO), 8-key
              // groups 1024 B apart (SBO); 16 keys = 2048 B per step.
              // A = P_gr: group gr wrote its bf16 pairs over the first 32 of its own 64 S
              // columns, [64 gr, 64 gr + 32), 8 columns per 16 keys
              const uint64_t bdesc = umma_desc_sw128(vb + kk * 2048, kBoxBytes, 1024);
              umma_ts(tmem + kColO + 128 * gr, tmem + col_s(s) + 64 * gr + (kk - 4 * gr) * 8,
                      bdesc, idesc_pv, (j > 0 || kk > 4 * gr) ? 1u : 0u);
            }
          }
          if (!ok) break;
          umma_commit(&v_empty[vs]);
          // one completion barrier per S buffer keeps every waiter within one phase of it
          umma_commit(&pv_done[s]);
        }
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, a.status);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    // Two warpgroups share the 128 rows: warp w reads TMEM lanes 32*(w%4).., group g owns
    // the 64 score columns [64g, 64g+64) of every row with its own running max m_g, sum
    // l_g and accumulator O_g (= P[:, 64g:64g+64] V[64g:64g+64, :]), so the groups never
    // wait for each other inside the loop; the epilogue combines the two halves once.
    const int wg = threadIdx.x >> 7;
    const int r = threadIdx.x & 127;  // row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t cs0 = static_cast<uint32_t>(kCols * wg);  // S column offset
    const uint32_t og = kColO + 128u * wg;                    // this group's O_g
    float* red = reinterpret_cast<float*>(tmem_slot + 4);     // [2 parity][kGroups][2][128]
    const float sl2 = a.scale_log2;
    const uint64_t sl2x2 = pack_f32x2(sl2, sl2);
    bool ok = true;
    int64_t g = 0;
    int li = 0;
    // plan offsets and first entry of this CTA's next item, loaded ahead (during the previous
    // item's epilogue) so that a new item does not start with two dependent global loads
    int nx_e0 = 0, nx_n = 0;
    int2 nx_ent = make_int2(0, 0);
    auto fetch_item = [&](int64_t itn) {
      if (itn >= n_items) return;
      int qt, b, head;
      item_of(itn, qt, b, head);
      nx_e0 = a.off[qt];
      nx_n = a.off[qt + 1] - nx_e0;
      nx_ent = nx_n > 0 ? reinterpret_cast<const int2*>(a.ent)[nx_e0] : make_int2(0, 0);
    };
    fetch_item(blockIdx.x);
    for (int64_t it = blockIdx.x; it < n_items; it += gridDim.x, ++li) {
      int qt, b, head;
      item_of(it, qt, b, head);
      const int e0 = nx_e0;
      const int n = nx_n;
      const int64_t row = (int64_t)qt * kBq + r;
      float m = -INFINITY;  // running max of raw scores (softmax scale > 0 keeps the order)
      float l = 0.f;
      int2 ent_next = nx_ent;
      for (int j = 0; j < n; ++j, ++g) {
        const int s = static_cast<int>(g & 1);
        const int kt = ent_next.x;
        const int flag = ent_next.y;
        if (j + 1 < n) ent_next = reinterpret_cast<const int2*>(a.ent)[e0 + j + 1];
        // warp-uniform outcome: the tcgen05.ld/st below are warp-collective
        ok = ok && __all_sync(0xffffffffu, mbar_wait(&s_full[s],
                                                      static_cast<uint32_t>((g >> 1) & 1),
                                                      a.status));
        if (!ok) continue;  // keep iterating: every warp must reach the epilogue barriers
        tc_fence_after();
        float x[kCols];
        {
          // both 32-column loads in flight before one wait
          uint32_t raw[kCols / 32][32];
#pragma unroll
          for (int c = 0; c < kCols / 32; ++c)
            tmem_ld32(lane_base + col_s(s) + cs0 + 32 * c, raw[c]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < kCols / 32; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i) x[32 * c + i] = __uint_as_float(raw[c][i]);
        }
        if (flag == PS_TILE_PARTIAL) {
          // visible keys of this row inside the slice: two intervals, as a 64-bit mask
          const uint64_t vis = visible_bits(row, (int64_t)kt * kBk + cs0, a.seq, a.lp, a.w);
          const uint32_t vlo = static_cast<uint32_t>(vis), vhi = static_cast<uint32_t>(vis >> 32);
#pragma unroll
          for (int i = 0; i < kCols; ++i) {
            const uint32_t word = i < 32 ? vlo : vhi;
            if (!(word & (1u << (i & 31)))) x[i] = -INFINITY;
          }
        }
        float t8[kCols / 4];
#pragma unroll
        for (int i = 0; i < kCols / 4; ++i)
          t8[i] = max3f(x[4 * i], x[4 * i + 1], fmaxf(x[4 * i + 2], x[4 * i + 3]));
#pragma unroll
        for (int n2 = kCols / 4; n2 > 1; n2 = (n2 + 1) / 2) {
#pragma unroll
          for (int i = 0; i < n2 / 2; ++i) t8[i] = fmaxf(t8[2 * i], t8[2 * i + 1]);
          if (n2 & 1) t8[n2 / 2] = t8[n2 - 1];
        }
        const float m_new = fmaxf(m, t8[0]);
        // Rescale O_g (and l) when the max of some row of this warp grew by more than 2^8.
        if (__any_sync(0xffffffffu, (m_new - m) * sl2 > kRescaleThreshold)) {
          float f = 1.f;
          if (m_new != -INFINITY) f = (m == -INFINITY) ? 0.f : fast_exp2((m - m_new) * sl2);
          if (j > 0) {
            // O_g holds this item's PVs up to tile g-1: wait for it, then scale in place
            const int64_t gp = g - 1;
            if (__all_sync(0xffffffffu, mbar_wait(&pv_done[gp & 1],
                                                  static_cast<uint32_t>((gp >> 1) & 1),
                                                  a.status))) {
              tc_fence_after();
              const uint64_t f2 = pack_f32x2(f, f);
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(lane_base + og + 32 * c, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const uint64_t v = fmul2(pack_f32x2(__uint_as_float(o[2 * i]),
                                                      __uint_as_float(o[2 * i + 1])), f2);
                  const float2 w2 = unpack_f32x2(v);
                  o[2 * i] = __float_as_uint(w2.x);
                  o[2 * i + 1] = __float_as_uint(w2.y);
                }
                tmem_st32(lane_base + og + 32 * c, o);
              }
              tmem_wait_st();
            } else {
              ok = false;
              continue;
            }
          }
          l *= f;
          if (m_new != -INFINITY) m = m_new;
        }
        // p = 2^(x * scale*log2e - m * scale*log2e), two lanes per instruction
        const float ms = (m == -INFINITY) ? 0.f : m * sl2;
        const uint64_t nms2 = pack_f32x2(-ms, -ms);
        uint64_t acc0 = pack_f32x2(0.f, 0.f), acc1 = acc0;
        // P over this group's own S columns (the other group may not have read its scores),
        // published in two halves of 32 keys: the PV products of the first half run while
        // the second half's exponentials are formed
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[kCols / 4];
#pragma unroll
          for (int ii = 0; ii < kCols / 4; ++ii) {
            const int i = hf * (kCols / 4) + ii;
            const float2 e =
                unpack_f32x2(ffma2(pack_f32x2(x[2 * i], x[2 * i + 1]), sl2x2, nms2));
            const float p0 = fast_exp2(e.x), p1 = fast_exp2(e.y);
            if (i & 1)
              acc1 = fadd2(acc1, pack_f32x2(p0, p1));
            else
              acc0 = fadd2(acc0, pack_f32x2(p0, p1));
            pk[ii] = cvt_bf16x2(p0, p1);
          }
          tmem_st16(lane_base + col_s(s) + cs0 + 16 * hf, pk);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_ready[(s * kGroups + wg) * 2 + hf]);
        }
        const float2 a0 = unpack_f32x2(acc0), a1 = unpack_f32x2(acc1);
        l += (a0.x + a0.y) + (a1.x + a1.y);
      }
      // ---------------------------------------------------------- epilogue of the item
      fetch_item(it + gridDim.x);
      // O = (2^(m_0 - M) O_0 + 2^(m_1 - M) O_1) / (2^(m_0 - M) l_0 + 2^(m_1 - M) l_1)
      const bool fin = ok && n > 0 &&
                       mbar_wait(&pv_done[(g - 1) & 1], static_cast<uint32_t>(((g - 1) >> 1) & 1),
                                 a.status);
      float* rd = red + (li & 1) * (kGroups * 2 * 128);
      rd[(wg * 2 + 0) * 128 + r] = m;
      rd[(wg * 2 + 1) * 128 + r] = l;
      const bool all_fin = named_bar_and(1, kSoftmaxThreads, fin);
      ok = ok && all_fin;
      if (all_fin) {
        tc_fence_after();
        const float m0 = rd[0 * 128 + r], l0 = rd[1 * 128 + r];
        const float m1 = rd[2 * 128 + r], l1 = rd[3 * 128 + r];
        const float M = fmaxf(m0, m1);
        const float f0 = (m0 == -INFINITY) ? 0.f : fast_exp2((m0 - M) * sl2);
        const float f1 = (m1 == -INFINITY) ? 0.f : fast_exp2((m1 - M) * sl2);
        const float lt = f0 * l0 + f1 * l1;
        const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
        const float g0 = f0 * inv_l, g1 = f1 * inv_l;
        uint32_t oa[2][32], ob[2][32];
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) {
          tmem_ld32(lane_base + kColO + cs0 + 32 * c, oa[c]);
          tmem_ld32(lane_base + kColO + 128 + cs0 + 32 * c, ob[c]);
        }
        tmem_wait_ld();
        // O is in registers: the next item's first PV may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);
        const bool store = row < a.seq;
        // this row's 64 outputs as 8 chunks of 8 bf16
        uint4 ch[8];
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = cvt_bf16x2(
                g0 * __uint_as_float(oa[c][2 * i]) + g1 * __uint_as_float(ob[c][2 * i]),
                g0 * __uint_as_float(oa[c][2 * i + 1]) + g1 * __uint_as_float(ob[c][2 * i + 1]));
#pragma unroll
          for (int v = 0; v < 4; ++v)
            ch[4 * c + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
        // Rows are a head stride apart in `out`, so one row per lane would make every store
        // instruction touch 32 lines.  Transpose 8 x 8 chunk blocks across each 8-lane group
        // (lane 8q + i then holds chunk i of rows 8q .. 8q + 7) so that each instruction
        // writes 4 whole 128-byte row slices.
        const int i8 = lane & 7;
#pragma unroll
        for (int d = 4; d > 0; d >>= 1) {
          const bool hi = (i8 & d) != 0;
#pragma unroll
          for (int j0 = 0; j0 < 8; ++j0) {
            if (j0 & d) continue;
            const uint4 snd = hi ? ch[j0] : ch[j0 | d];
            uint4 rcv;
            rcv.x = __shfl_xor_sync(0xffffffffu, snd.x, d);
            rcv.y = __shfl_xor_sync(0xffffffffu, snd.y, d);
            rcv.z = __shfl_xor_sync(0xffffffffu, snd.z, d);
            rcv.w = __shfl_xor_sync(0xffffffffu, snd.w, d);
            if (hi)
              ch[j0] = rcv;
            else
              ch[j0 | d] = rcv;
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int64_t rk = (int64_t)qt * kBq + 32 * (warp & 3) + (lane & ~7) + k;
          if (rk < a.seq)
            *reinterpret_cast<uint4*>(
                a.out + (((int64_t)b * a.seq + rk) * a.hq + head) * kHeadDim + cs0 + 8 * i8) =
                ch[k];
        }
        if (store && wg == 0 && a.lse)
          a.lse[((int64_t)b * a.hq + head) * a.seq + row] =
              lt > 0.f ? (M * sl2 + log2f(lt)) * kLn2 : -INFINITY;
      }
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
    rc = check_cuda(cudaFuncSetAttribute(prefill_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes),
                    "cudaFuncSetAttribute(prefill_kernel)");
    if (rc != PS_OK) return rc;
    attr_set[dev] = true;
  }
  const int64_t items = l.batch * l.hq * nq;
  if (items <= 0) return PS_OK;
  if (items > 0x7fffffffLL) return fail(PS_ERR_UNSUPPORTED, "prefill problem too large");
  // persistent: one CTA per SM walks items blockIdx.x, blockIdx.x + grid, ...
  const int64_t grid = items < sm_count() ? items : sm_count();
  return check_cuda(launch_pdl(prefill_kernel, dim3(static_cast<unsigned>(grid)), dim3(kThreads),
                               kSmemBytes, stream, mq, mk, mv, a),
                    "prefill_kernel launch");
}

}  // namespace ps
