// Masked prefill (truncated-backprop context forward) for Prefix Sliding, sm_100a:
// the device tile planner.  The attention kernel itself lives in ps_prefill_attn.cu.
//
// Two-level filtering ("Prefix Sliding 完全拆解", §Kernel 实现): key tiles wholly inside the
// evicted region are dropped at schedule time and never loaded; boundary tiles are masked
// element-wise; every other tile runs unmasked.  The planner writes, per query tile, the
// ascending list of (k_tile, flag) the attention kernel walks: the prefix tiles first,
// then the window tiles.
#include <cuda_runtime.h>

#include "ps_device.cuh"
#include "ps_internal.h"
#include "ps_ranges.cuh"

namespace ps {

namespace {
constexpr int kPlanThreads = 1024;

// Single-CTA planner (32 warps): the tiles per query tile in closed form, an exclusive scan
// of those counts into offsets (warp shuffles, then the warp totals), then one warp per query
// tile writes its entries, 32 candidate key tiles at a time, compacted by a ballot in
// ascending order.  ws_off: [nq + 1] int32; ws_ent: [n_tiles][2] int32 (k_tile, flag);
// plan_out (optional): [n_tiles][3] int32 (q_tile, k_tile, flag).
__global__ void __launch_bounds__(kPlanThreads)
    plan_kernel(int64_t seq, int32_t lp, int32_t w, int32_t* __restrict__ ws_off,
                int32_t* __restrict__ ws_ent, int32_t* __restrict__ plan_out) {
  constexpr int kWarps = kPlanThreads / 32;
  static_assert(kWarps == 32, "the warp totals are scanned by one warp");
  __shared__ int32_t s_warp[kWarps];
  __shared__ int32_t s_base;
  pdl_trigger();  // the attention kernel may start its prologue; it waits for this plan
  const int64_t nq = (seq + kPrefillBq - 1) / kPrefillBq;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) s_base = 0;
  __syncthreads();
  for (int64_t c0 = 0; c0 < nq; c0 += kPlanThreads) {
    const int64_t qt = c0 + threadIdx.x;
    const int32_t cnt =
        qt < nq ? static_cast<int32_t>(qtile_count(qt, seq, lp, w, kPrefillBq, kPrefillBk)) : 0;
    int32_t v = cnt;  // inclusive scan inside the warp
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += u;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int32_t t = s_warp[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, t, off);
        if (lane >= off) t += u;
      }
      s_warp[lane] = t;  // inclusive totals of warps 0 .. lane
    }
    __syncthreads();
    const int32_t base = s_base;
    if (qt < nq) ws_off[qt] = base + (warp > 0 ? s_warp[warp - 1] : 0) + v - cnt;
    __syncthreads();
    if (threadIdx.x == 0) s_base = base + s_warp[kWarps - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) ws_off[nq] = s_base;
  __syncthreads();  // the offsets are visible to every warp of the block
  const int64_t kt_last = (seq - 1) / kPrefillBk;
  for (int64_t qt = warp; qt < nq; qt += kWarps) {
    int64_t pe, wsb, we;
    qtile_candidates(qt, seq, lp, w, kPrefillBq, kPrefillBk, &pe, &wsb, &we);
    int32_t k = ws_off[qt];
    for (int pass = 0; pass < 2; ++pass) {
      const int64_t lo = pass == 0 ? 0 : wsb;
      const int64_t hi = pass == 0 ? (pe - 1 < kt_last ? pe - 1 : kt_last) : we;
      for (int64_t k0 = lo; k0 <= hi; k0 += 32) {  // warp-uniform bounds
        const int64_t kt = k0 + lane;
        const int32_t f =
            kt <= hi ? classify_tile(qt, kt, seq, lp, w, kPrefillBq, kPrefillBk) : 0;
        const unsigned m = __ballot_sync(0xffffffffu, f != 0);
        if (f) {
          const int32_t e = k + __popc(m & ((1u << lane) - 1u));
          ws_ent[2 * e] = static_cast<int32_t>(kt);
          ws_ent[2 * e + 1] = f;
          if (plan_out) {
            plan_out[3 * e] = static_cast<int32_t>(qt);
            plan_out[3 * e + 1] = static_cast<int32_t>(kt);
            plan_out[3 * e + 2] = f;
          }
        }
        k += __popc(m);
      }
    }
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
}  // namespace

int64_t prefill_plan_tiles(int64_t seq, int32_t lp, int32_t w) {
  const int64_t nq = (seq + kPrefillBq - 1) / kPrefillBq;
  int64_t total = 0;
  for (int64_t qt = 0; qt < nq; ++qt) total += qtile_count(qt, seq, lp, w, kPrefillBq, kPrefillBk);
  return total;
}

// Workspace: [plan offsets][plan entries][attention-kernel scratch].
size_t prefill_plan_bytes(int64_t seq, int64_t n_tiles) {
  const int64_t nq = (seq + kPrefillBq - 1) / kPrefillBq;
  return align256(size_t(nq + 1) * 4) + align256(size_t(n_tiles) * 8);
}

cudaError_t launch_plan(int64_t seq, int32_t lp, int32_t w, int64_t n_tiles, void* workspace,
                        int32_t* plan_out, cudaStream_t stream) {
  const int64_t nq = (seq + kPrefillBq - 1) / kPrefillBq;
  int32_t* off = static_cast<int32_t*>(workspace);
  int32_t* ent = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) +
                                            align256(size_t(nq + 1) * 4));
  (void)n_tiles;
  plan_kernel<<<1, kPlanThreads, 0, stream>>>(seq, lp, w, off, ent, plan_out);
  return cudaGetLastError();
}

}  // namespace ps
