// 3D-RoPE kernels of the bf16 path [paperlayer App. C.1, App. D.3, App. D.5]:
//  * rope_window_bf16: rotate every positional key of the window with its
//    window-relative (t, h, w) into the workspace (bf16, or fp16 for the per-head
//    keys of reconstruct-once).  HBM-bound: each thread moves one 16-byte vector
//    (4 rotary pairs) in and out, fully coalesced.
//  * dense_q_bf16: the dense path's query [q_nope | RoPE(q_rope)], re-laid out
//    head-major for the attention kernel's TMA tiles, in bf16 (the dense cache) or fp16 (the
//    reconstruct-once workspace).
#include <cuda_fp16.h>

#include "kernels.h"
#include "rope.cuh"

namespace vmla {
namespace {

constexpr int kMaxHeads16 = 1024;  // threads of a per-head query block: 16 per head, up to 64 heads

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// d_rope / 8 threads per key slot, 16 bytes (4 rotary pairs) each; a thread takes its slot in
// every sample, so the (cos, sin) of its 4 pairs are computed once for the batch.  The stored
// bf16 keys are rotated and written as bf16.
__global__ void __launch_bounds__(256) rope_window_bf16_kernel(const RopeWindow a) {
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int nq = a.d_rope >> 3;  // 16-byte pieces of a key
  if (idx >= (int64_t)a.n_keys * nq) return;
  const int quad = (int)(idx % nq);
  const int s = (int)(idx / nq);
  const int64_t ring_rows = (int64_t)a.ring.window_frames * a.ring.tokens_per_frame;
  const int fslot = s / a.ring.tokens_per_frame, tok = s % a.ring.tokens_per_frame;
  const int t = ring_slot_t(a.ring, fslot, a.window_start_slot);
  const int hh = tok / a.ring.grid_w, ww = tok % a.ring.grid_w;
  float2 cs[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) cs[k] = rope_cs(a.rope, quad * 4 + k, t, hh, ww);
  const uint4* src =
      reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.kr) + (int64_t)s * a.d_rope + quad * 8);
  uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.kr_rot) + (int64_t)s * a.d_rope + quad * 8);
  const int64_t stride = ring_rows * nq;  // one sample's ring, in 16-byte units
  // up to 8 samples at a time: every load is issued before the first store
  for (int b0 = 0; b0 < a.batch; b0 += 8) {
    const int nb = min(8, a.batch - b0);
    uint4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < nb) v[k] = __ldg(src + (b0 + k) * stride);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k >= nb) break;
      uint32_t in[4] = {v[k].x, v[k].y, v[k].z, v[k].w}, out[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        float u = bf_lo(in[p]), x = bf_hi(in[p]);
        rope_apply(u, x, cs[p]);
        out[p] = pack2(u, x);
      }
      dst[(b0 + k) * stride] = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
}

// One block per (sample, query row): 16 threads per head, 8 dims each (n_heads * 16 threads).
// Those of the content dims copy them, those of the positional dims (the last d_rope of the 128)
// rotate them; the (cos, sin) of the row's rotary pairs are computed once for all heads.
__global__ void __launch_bounds__(kMaxHeads16) dense_q_bf16_kernel(const DenseQTc a) {
  __shared__ float2 cs[kMaxPairs];
  const int row = blockIdx.x;  // b * n_q + i
  const int i = row % a.n_q;
  const int tok = i % a.ring.tokens_per_frame;
  const int t = (int)(a.t_first + i / a.ring.tokens_per_frame);
  const int n_pairs = a.d_rope >> 1;
  for (int p = threadIdx.x; p < n_pairs; p += blockDim.x)
    cs[p] = rope_cs(a.rope, p, t, tok / a.ring.grid_w, tok % a.ring.grid_w);
  __syncthreads();
  const int chunk = threadIdx.x & 15;
  const int h = threadIdx.x >> 4;
  if (h >= a.n_heads) return;
  const int b = row / a.n_q;
  const __nv_bfloat16* src = a.q + ((int64_t)row * a.n_heads + h) * 128 + chunk * 8;
  const int64_t dst = (((int64_t)b * a.n_heads + h) * a.n_q + i) * 128 + chunk * 8;  // element offset
  const uint4 v = *reinterpret_cast<const uint4*>(src);
  const int first_rope_chunk = (128 - a.d_rope) >> 3;
  const bool rope = chunk >= first_rope_chunk;
  const int p0 = (chunk - first_rope_chunk) * 4;
  uint32_t in[4] = {v.x, v.y, v.z, v.w}, out[4];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float u = bf_lo(in[k]), x = bf_hi(in[k]);
    if (rope) rope_apply(u, x, cs[p0 + k]);
    amax = fmaxf(amax, fmaxf(fabsf(u), fabsf(x)));
    out[k] = a.f16 ? pack_h2(u, x) : pack2(u, x);
  }
  // fp16 out (the reconstruct-once workspace): the content dims convert exactly for bf16 values in
  // fp16's range; a value past it is reported
  if (a.f16 && !(amax <= 65504.f)) atomicOr(a.err, DEV_ERR_RANGE);
  uint4* d = a.f16 ? reinterpret_cast<uint4*>(static_cast<__half*>(a.qd) + dst)
                   : reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.qd) + dst);
  *d = make_uint4(out[0], out[1], out[2], out[3]);
}

}  // namespace

cudaError_t launch_rope_window_bf16(const RopeWindow& a, cudaStream_t s) {
  if (a.d_rope % 8 != 0 || a.d_rope <= 0 || a.d_rope > 2 * kMaxPairs) return cudaErrorInvalidValue;
  const int64_t total = (int64_t)a.n_keys * (a.d_rope / 8);
  if (total == 0 || a.batch == 0) return cudaSuccess;
  rope_window_bf16_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dense_q_bf16(const DenseQTc& a, cudaStream_t s) {
  if (a.d_rope <= 0 || a.d_rope > 128 || a.d_rope % 8 != 0 || (a.f16 && !a.err)) return cudaErrorInvalidValue;
  if (a.n_heads * 16 > kMaxHeads16) return cudaErrorInvalidValue;
  const int64_t rows = (int64_t)a.batch * a.n_q;
  if (rows == 0) return cudaSuccess;
  dense_q_bf16_kernel<<<(unsigned)rows, a.n_heads * 16, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace vmla
