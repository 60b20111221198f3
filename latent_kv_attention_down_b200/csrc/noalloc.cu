// Allocation-free chunk attention: the absorbed design of vmla_chunk_attention
// with its scratch (window positional keys rotated for this call, absorbed
// queries) held in a fixed array that lives in the library itself, for
// callers that cannot allocate device memory.
//
// The array is a file-scope __device__ variable of kNoallocScratchBytes: every
// GPU that loads this module holds it until the process exits.  Host code may
// not use the variable's name as a device address, so the first call on each
// device (with that device current) looks its address up with
// cudaGetSymbolAddress and keeps it; kernels get that pointer as an argument.
// The library's device status word is looked up the same way, once per device
// (device_error_word), so a later call makes no symbol lookup at all.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "kernels.h"
#include "vmla.h"

using namespace vmla;

namespace {

constexpr size_t kNoallocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};

// Device address of the array on the current device (looked up once per device).
vmla_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return VMLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return VMLA_ERR_CUDA;
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return VMLA_OK;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

}  // namespace

extern "C" vmla_status vmla_chunk_attention_noalloc(const vmla_config* cfg, int layer, const void* ckv,
                                                    const void* kr, int64_t frames_appended, const void* q,
                                                    const void* w_uk, const void* w_uv, void* out,
                                                    int64_t first_frame, int n_frames, void* stream) {
  vmla_status st = vmla_config_check(cfg);
  if (st != VMLA_OK) return st;
  const vmla_config& c = *cfg;
  if (c.dtype != VMLA_BF16) return VMLA_ERR_UNSUPPORTED_SHAPE;
  if (layer < 0 || layer >= c.layers) return VMLA_ERR_OUT_OF_RANGE;
  if (!aligned16(ckv) || !aligned16(kr) || !aligned16(q) || !aligned16(w_uk) || !aligned16(w_uv) || !aligned16(out))
    return VMLA_ERR_INVALID_ARG;
  const int64_t F = frames_appended;
  // the absorbed kernels: up to 256 latent dims, up to 192 with 64 or 96 rotary dims
  if (!attn_absorbed_supported(c.d_latent, c.d_rope)) return VMLA_ERR_UNSUPPORTED_SHAPE;
  if (n_frames < 1 || n_frames > c.chunk_frames) return VMLA_ERR_OUT_OF_RANGE;
  if (F < 1 || first_frame < 0 || first_frame + n_frames != F) return VMLA_ERR_STATE;
  const bool at_read = c.rope_mode == VMLA_ROPE_AT_READ;
  if (!at_read && F > 1024) return VMLA_ERR_OUT_OF_RANGE;

  const int64_t T = (int64_t)c.grid_h * c.grid_w;
  const int64_t rr = (int64_t)c.window_frames * T;
  // active context [paperlayer App. D.4, D.5]: sink frames, then the newest W - S frames
  const Window win = window_of(c, F);
  const int n_keys = win.n_keys;
  const int nq = (int)(n_frames * T);
  const int dqk = c.d_latent + c.d_rope;
  const size_t kr_rot_bytes = at_read ? align256((size_t)c.batch * rr * c.d_rope * 2) : 0;
  const size_t qt_bytes = (size_t)c.batch * c.n_heads * nq * dqk * 2;
  if (kr_rot_bytes + qt_bytes > kNoallocScratchBytes) return VMLA_ERR_OUT_OF_RANGE;

  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != VMLA_OK) return st;
  unsigned* err = device_error_word();
  if (!err) return VMLA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const Rope rope = make_rope(c);
  const Ring ring = make_ring(c);

  const size_t layer_rows = (size_t)layer * c.batch * rr;
  const __nv_bfloat16* ckv_layer = static_cast<const __nv_bfloat16*>(ckv) + layer_rows * c.d_latent;
  const __nv_bfloat16* kr_layer = static_cast<const __nv_bfloat16*>(kr) + layer_rows * c.d_rope;
  void* kr_rot = scratch;  // the window's positional keys rotated for this call (bf16)
  __nv_bfloat16* qt = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(scratch) + kr_rot_bytes);

  const void* kpos = kr_layer;
  if (at_read) {
    RopeWindow r{kr_layer, kr_rot, c.batch, n_keys, c.d_rope, win.start_slot, ring, rope};
    if (launch_rope_window_bf16(r, s) != cudaSuccess) return VMLA_ERR_CUDA;
    kpos = kr_rot;
  }
  const CUtensorMapSwizzle SW128 = CU_TENSOR_MAP_SWIZZLE_128B;
  CUtensorMap tq, tuk, tqt;
  if (!map3(&tq, q, (uint64_t)c.n_heads * 128, nq, c.batch, (uint64_t)c.n_heads * 256, (uint64_t)nq * c.n_heads * 256,
                64, 128, SW128) ||
      !map3(&tuk, w_uk, c.d_latent, c.d_nope, c.n_heads, (uint64_t)c.d_latent * 2,
            (uint64_t)c.d_nope * c.d_latent * 2, 64, c.d_nope, SW128) ||
      !map3(&tqt, qt, dqk, nq, (uint64_t)c.batch * c.n_heads, (uint64_t)dqk * 2, (uint64_t)nq * dqk * 2, 64, 64,
                SW128))
    return VMLA_ERR_CUDA;
  QPrepTc qa;
  qa.q = static_cast<const __nv_bfloat16*>(q);
  qa.qt = qt;
  qa.n_q = nq;
  qa.n_heads = c.n_heads;
  qa.d_latent = c.d_latent;
  qa.d_rope = c.d_rope;
  qa.t_first = first_frame - (at_read ? win.t_origin : 0);
  qa.ring = ring;
  qa.rope = rope;
  qa.err = err;
  qa.limit_ns = kWaitLimitNs;
  if (launch_qprep_tc(tq, tuk, tqt, qa, c.batch, s) != cudaSuccess) return VMLA_ERR_CUDA;

  const int bn = attn_absorbed_block_n(c.d_latent);
  // the rotary columns: one box d_rope wide swizzled at its row width, or three boxes of 32 for 96
  const int rbox = c.d_rope == 96 ? 32 : c.d_rope;
  const CUtensorMapSwizzle rsw = rbox == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                            : (rbox == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  const uint64_t bh = (uint64_t)c.batch * c.n_heads;
  CUtensorMap mq, mqr, mk, mkr, muv, mo;
  if (!map3(&mq, qt, dqk, nq, bh, (uint64_t)dqk * 2, (uint64_t)nq * dqk * 2, 64, 128, SW128) ||
      !map3(&mqr, qt, dqk, nq, bh, (uint64_t)dqk * 2, (uint64_t)nq * dqk * 2, rbox, 128, rsw) ||
      !map3(&mk, ckv_layer, c.d_latent, n_keys, c.batch, (uint64_t)c.d_latent * 2, (uint64_t)rr * c.d_latent * 2,
                64, bn, SW128) ||
      !map3(&mkr, kpos, c.d_rope, n_keys, c.batch, (uint64_t)c.d_rope * 2, (uint64_t)rr * c.d_rope * 2, rbox, bn,
            rsw) ||
      !map3(&muv, w_uv, c.d_latent, 128, c.n_heads, (uint64_t)c.d_latent * 2, 128ull * c.d_latent * 2, 64, 128,
                SW128) ||
      !map3(&mo, out, (uint64_t)c.n_heads * 128, nq, c.batch, (uint64_t)c.n_heads * 512,
                (uint64_t)nq * c.n_heads * 512, 32, 128, SW128, CU_TENSOR_MAP_DATA_TYPE_FLOAT32))
    return VMLA_ERR_CUDA;
  AttnTc a;
  a.n_q = nq;
  a.n_keys = n_keys;
  a.n_heads = c.n_heads;
  a.m_tiles = (nq + 127) / 128;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)(c.d_nope + c.d_rope)));
  a.rescale_threshold = c.softmax_rescale_log2;
  a.err = err;
  a.limit_ns = kWaitLimitNs;
  return launch_attn_absorbed_tc(c.d_latent, c.d_rope, mq, mqr, mk, mkr, muv, mo, a, c.batch, s) == cudaSuccess
             ? VMLA_OK
             : VMLA_ERR_CUDA;
}
