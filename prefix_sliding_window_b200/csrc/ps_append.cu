// KV append with Continue-PE RoPE into the Prefix Sliding store, sm_100a.
//
// "Prefix Sliding 完全拆解", §位置编码 (Continue PE): every token keeps its absolute position
// id, so a key is rotated exactly once, when it is cached, and reused as is afterwards.
// §核心机制: the store per sequence is bounded by L_prefix + W; a token past the prefix
// overwrites the ring slot (pos - L_prefix) mod W, evicting the position it held.
//
// One CTA per appended token (sequence b, token t, position p = pos0[b] + t):
//  * threads 0..63 form the 64 RoPE angles p * theta^(-2i/128) in float64 (at p ~ 2^18 an
//    fp32 product would already be off by ~0.03 rad; the host supplies theta^(-2i/128) in
//    float64), reduce them modulo 2*pi in float64 and keep cos/sin in fp32 in shared memory;
//  * every thread rotates 8 rotate-half pairs at a time (16-byte loads of x1 and x2),
//    writes rotated K and the V row to the prefix row or ring slot, and rotates q in place.
// When several of the T tokens fall on one ring slot only the latest is written, so the
// result does not depend on thread scheduling.
#include <cuda_bf16.h>
#include <math.h>

#include "ps_device.cuh"
#include "ps_internal.h"

namespace ps {
namespace {

constexpr int kAppendThreads = 256;
constexpr int kHalf = kHeadDim / 2;  // rotate-half pairs per head
constexpr int kChunks = kHalf / 8;   // 16-byte chunks per half

__device__ __forceinline__ void rotate8(const uint4& x1, const uint4& x2, const float* cs,
                                        const float* sn, uint4& y1, uint4& y2) {
  const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(&x1);
  const __nv_bfloat162* bb = reinterpret_cast<const __nv_bfloat162*>(&x2);
  __nv_bfloat162* o1 = reinterpret_cast<__nv_bfloat162*>(&y1);
  __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&y2);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 u = __bfloat1622float2(a[e]);
    const float2 v = __bfloat1622float2(bb[e]);
    const float c0 = cs[2 * e], c1 = cs[2 * e + 1];
    const float s0 = sn[2 * e], s1 = sn[2 * e + 1];
    o1[e] = __floats2bfloat162_rn(rope_lo(u.x, v.x, c0, s0), rope_lo(u.y, v.y, c1, s1));
    o2[e] = __floats2bfloat162_rn(rope_hi(u.x, v.x, c0, s0), rope_hi(u.y, v.y, c1, s1));
  }
}

__global__ void __launch_bounds__(kAppendThreads) append_rope_kernel(const AppendArgs a) {
  // Launched with programmatic serialization: wait for the previous kernel in the stream
  // (inputs may come from it) before reading anything, then let the decode that usually
  // follows start its prologue (it reads q and the newest row only after this grid ends).
  pdl_wait();
  pdl_trigger();
  __shared__ float s_cos[kHalf];
  __shared__ float s_sin[kHalf];
  const int64_t tok = blockIdx.x;
  const int64_t b = tok / a.T;
  const int t = static_cast<int>(tok % a.T);
  const int64_t p0 = a.pos0[b];
  const int64_t p = p0 + t;
  const int64_t p_last = p0 + a.T - 1;

  if (p < 0) {
    if (threadIdx.x == 0 && a.status) atomicOr(a.status, PS_DEV_BAD_POS);
    return;
  }
  const bool linear = (a.k_ring == nullptr);
  if (linear && p >= a.lp) {
    if (threadIdx.x == 0 && a.status) atomicOr(a.status, PS_DEV_POS_RANGE);
    return;
  }
  // where this token's K/V row goes (or nowhere, if a later token of this call owns it)
  const __nv_bfloat16* k_src = static_cast<const __nv_bfloat16*>(a.k_new) + tok * a.hkv * kHeadDim;
  const __nv_bfloat16* v_src = static_cast<const __nv_bfloat16*>(a.v_new) + tok * a.hkv * kHeadDim;
  __nv_bfloat16* k_dst_base = nullptr;
  __nv_bfloat16* v_dst_base = nullptr;
  int64_t row_stride_rows = 0, row = 0;
  if (p < a.lp && a.k_pre == nullptr) {
    // ring-only cache (the prefix lives elsewhere, e.g. shared by a group of sequences)
    if (threadIdx.x == 0 && a.status) atomicOr(a.status, PS_DEV_POS_RANGE);
    return;
  }
  if (p < a.lp) {
    k_dst_base = static_cast<__nv_bfloat16*>(a.k_pre);
    v_dst_base = static_cast<__nv_bfloat16*>(a.v_pre);
    row_stride_rows = a.lp;
    row = p;
  } else if (p > p_last - a.w) {
    k_dst_base = static_cast<__nv_bfloat16*>(a.k_ring);
    v_dst_base = static_cast<__nv_bfloat16*>(a.v_ring);
    row_stride_rows = a.w;
    row = (p - a.lp) % a.w;
  }
  int64_t blk = b;  // the store's (sequence or pool block) index in its outermost dimension
  if (a.paged && k_dst_base) {
    // 64-row blocks of the pool: logical block row / 64 (prefix) or pre_blocks + slot / 64
    const int64_t lb = (p < a.lp ? 0 : a.pre_blocks) + row / 64;
    blk = a.table[b * a.table_stride + lb];
    row_stride_rows = 64;
    row %= 64;
    if (blk < 0 || blk >= a.n_blocks) {  // a bad table entry: flag it, write nothing
      if (threadIdx.x == 0 && a.status) atomicOr(a.status, PS_DEV_POS_RANGE);
      k_dst_base = v_dst_base = nullptr;
    }
  }
  __nv_bfloat16* qb = static_cast<__nv_bfloat16*>(a.q) + tok * a.hq * kHeadDim;

  // Work items: K rotate (hkv x kChunks), V copy (hkv x 16), q rotate (hq x kChunks).
  const int n_k = k_dst_base ? a.hkv * kChunks : 0;
  const int n_v = k_dst_base ? a.hkv * (kHeadDim / 8) : 0;
  const int n_q = a.q ? a.hq * kChunks : 0;
  const int n_items = n_k + n_v + n_q;
  auto load = [&](int it, uint4& x1, uint4& x2) {
    if (it < n_k) {
      const __nv_bfloat16* src = k_src + (it / kChunks) * kHeadDim + 8 * (it % kChunks);
      x1 = *reinterpret_cast<const uint4*>(src);
      x2 = *reinterpret_cast<const uint4*>(src + kHalf);
    } else if (it < n_k + n_v) {
      const int j = it - n_k;
      x1 = *reinterpret_cast<const uint4*>(v_src + (j / 16) * kHeadDim + 8 * (j % 16));
    } else {
      const int j = it - n_k - n_v;
      const __nv_bfloat16* src = qb + (j / kChunks) * kHeadDim + 8 * (j % kChunks);
      x1 = *reinterpret_cast<const uint4*>(src);
      x2 = *reinterpret_cast<const uint4*>(src + kHalf);
    }
  };
  // the first item's inputs are fetched before the angles, so both latencies overlap
  uint4 x1 = make_uint4(0, 0, 0, 0), x2 = x1;
  if (threadIdx.x < n_items) load(threadIdx.x, x1, x2);

  if (threadIdx.x < kHalf) {
    // angle = p * inv_f[i], formed and reduced modulo 2 pi in float64 (rope_cos_sin)
    const float2 cs = rope_cos_sin(double(p), a.inv_freq[threadIdx.x]);
    s_cos[threadIdx.x] = cs.x;
    s_sin[threadIdx.x] = cs.y;
  }
  __syncthreads();

  for (int it = threadIdx.x; it < n_items; it += blockDim.x) {
    if (it != threadIdx.x) load(it, x1, x2);
    if (it < n_k) {
      const int h = it / kChunks, c = it % kChunks;
      uint4 y1, y2;
      rotate8(x1, x2, s_cos + 8 * c, s_sin + 8 * c, y1, y2);
      __nv_bfloat16* dst = k_dst_base + ((blk * a.hkv + h) * row_stride_rows + row) * kHeadDim;
      *reinterpret_cast<uint4*>(dst + 8 * c) = y1;
      *reinterpret_cast<uint4*>(dst + kHalf + 8 * c) = y2;
    } else if (it < n_k + n_v) {
      const int j = it - n_k;
      const int h = j / 16, c = j % 16;
      __nv_bfloat16* dst = v_dst_base + ((blk * a.hkv + h) * row_stride_rows + row) * kHeadDim;
      *reinterpret_cast<uint4*>(dst + 8 * c) = x1;
    } else {
      // q rotated in place at the token's own absolute position
      const int j = it - n_k - n_v;
      const int h = j / kChunks, c = j % kChunks;
      uint4 y1, y2;
      rotate8(x1, x2, s_cos + 8 * c, s_sin + 8 * c, y1, y2);
      __nv_bfloat16* dst = qb + h * kHeadDim;
      *reinterpret_cast<uint4*>(dst + 8 * c) = y1;
      *reinterpret_cast<uint4*>(dst + kHalf + 8 * c) = y2;
    }
  }
}

// Whether sequence b's promotion request is valid: inside the window of the latest position,
// after the last promoted token (ascending order), within capacity.  Both pin kernels
// evaluate it on the same inputs (pin_count changes only in the second).
__device__ __forceinline__ bool pin_valid(const PinArgs& a, int64_t b, int64_t* m_out,
                                          int32_t* cnt_out) {
  const int64_t t0 = a.t0[b], t1 = a.t1[b], p = a.pos[b];
  const int32_t cnt = a.pin_count[b];
  const int64_t m = t1 - t0;
  const int32_t cap = a.lcap - a.lp;
  *m_out = m;
  *cnt_out = cnt;
  if (m <= 0) return false;
  const int64_t* pp = a.pin_pos + b * cap;
  return t0 >= a.lp && t1 - 1 <= p && t0 > p - a.w && cnt + m <= cap &&
         (cnt == 0 || t0 > pp[cnt - 1]);
}

constexpr int kPinTokens = 32;  // tokens per copy block (one warp per token, 8 warps)

// Block (b, chunk) copies tokens [32 chunk, 32 chunk + 32) of sequence b's range: K and V
// rows from ring slots (t - lp) mod w to prefix rows lp + pin_count + (t - t0), 16 bytes per
// lane, and records their positions.  Keys stay as cached (Continue PE rotated them at their
// absolute positions already).
__global__ void __launch_bounds__(256) pin_copy_kernel(const PinArgs a) {
  const int64_t b = blockIdx.x;
  int64_t m;
  int32_t cnt;
  if (!pin_valid(a, b, &m, &cnt)) return;
  const int64_t first = (int64_t)blockIdx.y * kPinTokens;
  if (first >= m) return;
  const int n = static_cast<int>(m - first < kPinTokens ? m - first : kPinTokens);
  const int64_t t0 = a.t0[b] + first;
  constexpr int kChunks = kHeadDim / 8;  // 16-byte chunks per row
  const int per_token = a.hkv * 2 * kChunks;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = warp; i < n; i += 8) {
    const int64_t slot = (t0 + i - a.lp) % a.w;
    const int64_t row = a.lp + cnt + first + i;
    for (int j = lane; j < per_token; j += 32) {
      const int c = j % kChunks;
      const int kv = (j / kChunks) & 1;
      const int h = j / (2 * kChunks);
      const int64_t bh = b * a.hkv + h;
      const uint4* src = static_cast<const uint4*>(kv ? a.v_ring : a.k_ring) +
                         (bh * a.w + slot) * kChunks + c;
      uint4* dst = static_cast<uint4*>(kv ? a.v_pre : a.k_pre) + (bh * a.lcap + row) * kChunks + c;
      *dst = *src;
    }
  }
  if (threadIdx.x < n) a.pin_pos[b * (a.lcap - a.lp) + cnt + first + threadIdx.x] = t0 + threadIdx.x;
}

// One thread per sequence: advance pin_count (or flag an invalid request).
__global__ void pin_commit_kernel(const PinArgs a) {
  const int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= a.batch) return;
  int64_t m;
  int32_t cnt;
  if (pin_valid(a, b, &m, &cnt)) {
    a.pin_count[b] = cnt + static_cast<int32_t>(m);
  } else if (m > 0 && a.status) {
    atomicOr(a.status, PS_DEV_POS_RANGE);
  }
}

}  // namespace

cudaError_t launch_pin(const PinArgs& a, cudaStream_t stream) {
  if (a.batch <= 0) return cudaSuccess;
  if (a.batch > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const int64_t chunks = (a.lcap - a.lp + kPinTokens - 1) / kPinTokens;
  if (chunks > 65535) return cudaErrorInvalidConfiguration;
  pin_copy_kernel<<<dim3(static_cast<unsigned>(a.batch), static_cast<unsigned>(chunks)), 256, 0,
                    stream>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pin_commit_kernel<<<static_cast<unsigned>((a.batch + 255) / 256), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  const int64_t tokens = a.batch * a.T;
  if (tokens <= 0) return cudaSuccess;
  if (tokens > 0x7fffffff) return cudaErrorInvalidConfiguration;
  return launch_pdl(append_rope_kernel, dim3(static_cast<unsigned>(tokens)),
                    dim3(kAppendThreads), 0, stream, a);
}

}  // namespace ps
