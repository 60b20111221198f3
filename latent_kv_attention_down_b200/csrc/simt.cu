// fp32 SIMT kernels: the same steps as the tcgen05 path for any shape, used for
// VMLA_FP32 handles.  They are plain CUDA (one thread per output element or a
// block per query row) and make no attempt at speed.
#include "kernels.h"
#include "rope.cuh"

namespace vmla {
namespace {

// Row m of a call (frames first_frame ..) -> ring row of its sample.
__device__ __forceinline__ int64_t ring_row(const Ring& g, int64_t first_frame, int m) {
  const int64_t f = first_frame + m / g.tokens_per_frame;
  return ring_frame_slot(g, f) * g.tokens_per_frame + (m % g.tokens_per_frame);
}

// ---- append: [c | k_R] = W_down x
__global__ void append_simt_kernel(const SimtAppend a) {
  const int n_pairs = a.d_rope / 2;
  const int width = a.d_latent + n_pairs;
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)a.batch * a.rows * width;
  if (idx >= total) return;
  const int j = idx % width;
  const int m = (idx / width) % a.rows;
  const int b = idx / ((int64_t)width * a.rows);
  const float* x = a.x + ((int64_t)b * a.rows + m) * a.d_model;
  const int64_t row = a.contiguous ? m : ring_row(a.ring, a.first_frame, m);
  if (j < a.d_latent) {
    const float* w = a.w_down + (int64_t)j * a.d_model;
    float acc = 0.f;
    for (int k = 0; k < a.d_model; ++k) acc = fmaf(x[k], w[k], acc);
    a.ckv[((int64_t)b * a.out_rows + row) * a.d_latent + j] = acc;
  } else {
    const int p = j - a.d_latent;
    const float* w0 = a.w_down + (int64_t)(a.d_latent + 2 * p) * a.d_model;
    const float* w1 = w0 + a.d_model;
    float u = 0.f, v = 0.f;
    for (int k = 0; k < a.d_model; ++k) {
      u = fmaf(x[k], w0[k], u);
      v = fmaf(x[k], w1[k], v);
    }
    if (a.rotate) {
      const int tok = m % a.ring.tokens_per_frame;
      const int t = (int)(a.first_frame + m / a.ring.tokens_per_frame);
      rope_apply(u, v, rope_cs(a.rope, p, t, tok / a.ring.grid_w, tok % a.ring.grid_w));
    }
    float* kr = a.kr + ((int64_t)b * a.out_rows + row) * a.d_rope + 2 * p;
    kr[0] = u;
    kr[1] = v;
  }
}

// ---- window rotation of the positional keys (one thread per pair)
__global__ void rope_window_f32_kernel(const RopeWindow a) {
  const int n_pairs = a.d_rope / 2;
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)a.batch * a.n_keys * n_pairs;
  if (idx >= total) return;
  const int p = idx % n_pairs;
  const int s = (idx / n_pairs) % a.n_keys;
  const int b = idx / ((int64_t)n_pairs * a.n_keys);
  const int64_t ring_rows = (int64_t)a.ring.window_frames * a.ring.tokens_per_frame;
  const int fslot = s / a.ring.tokens_per_frame, tok = s % a.ring.tokens_per_frame;
  const int t = ring_slot_t(a.ring, fslot, a.window_start_slot);
  const float* src = static_cast<const float*>(a.kr) + ((int64_t)b * ring_rows + s) * a.d_rope + 2 * p;
  float* dst = static_cast<float*>(a.kr_rot) + ((int64_t)b * ring_rows + s) * a.d_rope + 2 * p;
  float u = src[0], v = src[1];
  rope_apply(u, v, rope_cs(a.rope, p, t, tok / a.ring.grid_w, tok % a.ring.grid_w));
  dst[0] = u;
  dst[1] = v;
}

// ---- query preparation
__global__ void qprep_simt_kernel(const SimtQPrep a) {
  const int n_pairs = a.d_rope / 2;
  const int lead = a.absorb ? a.d_latent : a.d_nope;
  const int width = lead + a.d_rope;
  const int jw = lead + n_pairs;
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)a.batch * a.n_heads * a.n_q * jw;
  if (idx >= total) return;
  const int j = idx % jw;
  const int i = (idx / jw) % a.n_q;
  const int h = (idx / ((int64_t)jw * a.n_q)) % a.n_heads;
  const int b = idx / ((int64_t)jw * a.n_q * a.n_heads);
  const int dq = a.d_nope + a.d_rope;
  const float* q = a.q + (((int64_t)b * a.n_q + i) * a.n_heads + h) * dq;
  float* out = a.qt + (((int64_t)b * a.n_heads + h) * a.n_q + i) * width;
  if (j < lead) {
    if (a.absorb) {
      const float* w = a.w_uk + (int64_t)h * a.d_nope * a.d_latent + j;
      float acc = 0.f;
      for (int n = 0; n < a.d_nope; ++n) acc = fmaf(q[n], w[(int64_t)n * a.d_latent], acc);
      out[j] = acc;
    } else {
      out[j] = q[j];
    }
  } else {
    const int p = j - lead;
    const int tok = i % a.ring.tokens_per_frame;
    const int t = (int)(a.t_first + i / a.ring.tokens_per_frame);
    float u = q[a.d_nope + 2 * p], v = q[a.d_nope + 2 * p + 1];
    rope_apply(u, v, rope_cs(a.rope, p, t, tok / a.ring.grid_w, tok % a.ring.grid_w));
    out[lead + 2 * p] = u;
    out[lead + 2 * p + 1] = v;
  }
}

constexpr int kAttnThreads = 128;
constexpr int kMaxWidth = 1024;

__device__ float block_max(float v, float* red) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < kAttnThreads / 32; ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}
__device__ float block_sum(float v, float* red) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
  for (int w = 0; w < kAttnThreads / 32; ++w) r += red[w];
  __syncthreads();
  return r;
}

// ---- attention: one block per (query row, head, sample), online softmax over key blocks
__global__ void __launch_bounds__(kAttnThreads) attn_simt_kernel(const SimtAttn a) {
  __shared__ float sq[kMaxWidth];
  __shared__ float sacc[kMaxWidth];
  __shared__ float sp[kAttnThreads];
  __shared__ float red[kAttnThreads / 32];
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int dqk = a.dense ? a.d_value : a.d_latent + a.d_rope;
  const int dacc = a.dense ? a.d_value : a.d_latent;
  const float* q = a.qt + (((int64_t)b * a.n_heads + h) * a.n_q + i) * dqk;
  for (int c = tid; c < dqk; c += kAttnThreads) sq[c] = q[c];
  for (int c = tid; c < dacc; c += kAttnThreads) sacc[c] = 0.f;
  __syncthreads();
  const int64_t dense_row = 2LL * a.n_heads * a.d_value;
  float m = -INFINITY, l = 0.f;
  for (int k0 = 0; k0 < a.n_keys; k0 += kAttnThreads) {
    const int j = k0 + tid;
    float s = -INFINITY;
    if (j < a.n_keys) {
      float acc = 0.f;
      if (a.dense) {
        const float* k = a.key + ((int64_t)b * a.ring_rows + j) * dense_row + (int64_t)h * a.d_value;
        for (int c = 0; c < dqk; ++c) acc = fmaf(sq[c], k[c], acc);
      } else {
        const float* k = a.key + ((int64_t)b * a.ring_rows + j) * a.d_latent;
        const float* kp = a.kpos + ((int64_t)b * a.ring_rows + j) * a.d_rope;
        for (int c = 0; c < a.d_latent; ++c) acc = fmaf(sq[c], k[c], acc);
        for (int c = 0; c < a.d_rope; ++c) acc = fmaf(sq[a.d_latent + c], kp[c], acc);
      }
      s = acc * a.scale;
    }
    const float m_new = fmaxf(m, block_max(s, red));
    const float alpha = expf(m - m_new);
    const float p = (j < a.n_keys) ? expf(s - m_new) : 0.f;
    l = l * alpha + block_sum(p, red);
    sp[tid] = p;
    __syncthreads();
    const int nk = min(kAttnThreads, a.n_keys - k0);
    for (int c = tid; c < dacc; c += kAttnThreads) {
      float acc = sacc[c] * alpha;
      for (int jj = 0; jj < nk; ++jj) {
        const float* v = a.dense
                             ? a.key + ((int64_t)b * a.ring_rows + k0 + jj) * dense_row +
                                   (int64_t)(a.n_heads + h) * a.d_value
                             : a.key + ((int64_t)b * a.ring_rows + k0 + jj) * a.d_latent;
        acc = fmaf(sp[jj], v[c], acc);
      }
      sacc[c] = acc;
    }
    m = m_new;
    __syncthreads();
  }
  const float inv_l = 1.f / l;
  float* out = a.out + ((int64_t)b * a.n_q + i) * a.n_heads * a.d_value + (int64_t)h * a.d_value;
  for (int e = tid; e < a.d_value; e += kAttnThreads) {
    if (a.dense) {
      out[e] = sacc[e] * inv_l;
    } else {
      const float* w = a.w_uv + ((int64_t)h * a.d_value + e) * a.d_latent;
      float acc = 0.f;
      for (int c = 0; c < a.d_latent; ++c) acc = fmaf(w[c], sacc[c], acc);
      out[e] = acc * inv_l;
    }
  }
}

// ---- dense per-head entries from a chunk's latents
__global__ void dense_reconstruct_simt_kernel(const SimtDenseReconstruct a) {
  const int n_pairs = a.d_rope / 2;
  const int width = a.d_nope + n_pairs + a.d_value;
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)a.batch * a.rows * a.n_heads * width;
  if (idx >= total) return;
  const int j = idx % width;
  const int h = (idx / width) % a.n_heads;
  const int m = (idx / ((int64_t)width * a.n_heads)) % a.rows;
  const int b = idx / ((int64_t)width * a.n_heads * a.rows);
  const float* c = a.c + ((int64_t)b * a.rows + m) * a.d_latent;
  const int64_t ring_rows = (int64_t)a.ring.window_frames * a.ring.tokens_per_frame;
  const int64_t row = ring_row(a.ring, a.first_frame, m);
  float* kdst = a.dense + ((int64_t)b * ring_rows + row) * (2LL * a.n_heads * a.d_value) + (int64_t)h * a.d_value;
  float* vdst = kdst + (int64_t)a.n_heads * a.d_value;
  if (j < a.d_nope) {
    const float* w = a.w_uk + ((int64_t)h * a.d_nope + j) * a.d_latent;
    float acc = 0.f;
    for (int k = 0; k < a.d_latent; ++k) acc = fmaf(w[k], c[k], acc);
    kdst[j] = acc;
  } else if (j < a.d_nope + n_pairs) {
    const int p = j - a.d_nope;
    const float* r = a.r + ((int64_t)b * a.rows + m) * a.d_rope + 2 * p;
    const int tok = m % a.ring.tokens_per_frame;
    const int t = (int)(a.first_frame + m / a.ring.tokens_per_frame);
    float u = r[0], v = r[1];
    rope_apply(u, v, rope_cs(a.rope, p, t, tok / a.ring.grid_w, tok % a.ring.grid_w));
    kdst[a.d_nope + 2 * p] = u;
    kdst[a.d_nope + 2 * p + 1] = v;
  } else {
    const int e = j - a.d_nope - n_pairs;
    const float* w = a.w_uv + ((int64_t)h * a.d_value + e) * a.d_latent;
    float acc = 0.f;
    for (int k = 0; k < a.d_latent; ++k) acc = fmaf(w[k], c[k], acc);
    vdst[e] = acc;
  }
}

inline unsigned grid_for(int64_t total, int threads) { return (unsigned)((total + threads - 1) / threads); }

}  // namespace

cudaError_t launch_append_simt(const SimtAppend& a, cudaStream_t s) {
  const int64_t total = (int64_t)a.batch * a.rows * (a.d_latent + a.d_rope / 2);
  if (total == 0) return cudaSuccess;
  append_simt_kernel<<<grid_for(total, 256), 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_rope_window_f32(const RopeWindow& a, cudaStream_t s) {
  const int64_t total = (int64_t)a.batch * a.n_keys * (a.d_rope / 2);
  if (total == 0) return cudaSuccess;
  rope_window_f32_kernel<<<grid_for(total, 256), 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_qprep_simt(const SimtQPrep& a, cudaStream_t s) {
  const int lead = a.absorb ? a.d_latent : a.d_nope;
  const int64_t total = (int64_t)a.batch * a.n_heads * a.n_q * (lead + a.d_rope / 2);
  if (total == 0) return cudaSuccess;
  qprep_simt_kernel<<<grid_for(total, 256), 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(const SimtAttn& a, cudaStream_t s) {
  const int dqk = a.dense ? a.d_value : a.d_latent + a.d_rope;
  if (dqk > kMaxWidth || a.d_latent > kMaxWidth || a.d_value > kMaxWidth) return cudaErrorInvalidValue;
  if (a.n_q == 0) return cudaSuccess;
  attn_simt_kernel<<<dim3(a.n_q, a.n_heads, a.batch), kAttnThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dense_reconstruct_simt(const SimtDenseReconstruct& a, cudaStream_t s) {
  const int64_t total = (int64_t)a.batch * a.rows * a.n_heads * (a.d_nope + a.d_rope / 2 + a.d_value);
  if (total == 0) return cudaSuccess;
  dense_reconstruct_simt_kernel<<<grid_for(total, 256), 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace vmla
