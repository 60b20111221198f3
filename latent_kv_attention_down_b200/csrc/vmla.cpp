// Host side of libvmla.so: the C ABI declared in include/vmla.h.
//
// Validates every call, keeps the per-layer frame counters of the sliding
// window (a ring of window_frames frames: the first sink_frames frames keep
// their slots, later ones rotate FIFO through the rest [paperlayer App. D.4]),
// encodes the TMA tensor maps of each launch and enqueues the kernels on the
// caller's stream.  It allocates no device memory.
#include "vmla.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "kernels.h"

using namespace vmla;

namespace vmla {

// ---------------------------------------------------------------- host helpers (declared in kernels.h)
Rope make_rope(const vmla_config& c) {
  Rope r;
  std::memset(&r, 0, sizeof(r));
  int p = 0;
  for (int a = 0; a < 3; ++a) {
    const double base = c.rope_base_dims[a] > 0 ? c.rope_base_dims[a] : 2.0 * c.rope_pairs[a];
    for (int i = 0; i < c.rope_pairs[a]; ++i) r.freq[p++] = (float)std::pow((double)c.rope_theta, -2.0 * i / base);
  }
  r.n_t = c.rope_pairs[0];
  r.n_h = c.rope_pairs[1];
  r.n_w = c.rope_pairs[2];
  return r;
}

Ring make_ring(const vmla_config& c) {
  return Ring{(int)((int64_t)c.grid_h * c.grid_w), c.grid_w, c.window_frames, c.sink_frames};
}

// The active context after F frames [paperlayer App. D.4, D.5]: ring slots [0, n_keys / T_f);
// a local frame f has window-relative t = f - t_origin, a sink frame t = f.
Window window_of(const vmla_config& c, int64_t F) {
  const int64_t S = c.sink_frames, L = c.window_frames - c.sink_frames;
  Window w;
  if (F <= c.window_frames) {
    w.local_start = std::min<int64_t>(S, F);
    w.t_origin = 0;
    w.n_keys = (int)(F * ((int64_t)c.grid_h * c.grid_w));
    w.start_slot = 0;
  } else {
    w.local_start = F - L;
    w.t_origin = w.local_start - S;
    w.n_keys = (int)((int64_t)c.window_frames * ((int64_t)c.grid_h * c.grid_w));
    w.start_slot = (int)((w.local_start - S) % L);
  }
  return w;
}

// ---------------------------------------------------------------- TMA tensor maps
namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

bool have_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode != nullptr;
}
}  // namespace

// 3D map: dims (d0 innermost, d1, d2), byte strides s1, s2, box (b0, b1, 1); bf16 unless told otherwise
bool map3(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
          uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw, CUtensorMapDataType dt) {
  if (!have_encode()) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return g_encode(m, dt, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool map2(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t s1, uint32_t b0, uint32_t b1,
          CUtensorMapSwizzle sw) {
  if (!have_encode()) return false;
  cuuint64_t dims[2] = {d0, d1};
  cuuint64_t strides[1] = {s1};
  cuuint32_t box[2] = {b0, b1};
  cuuint32_t es[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace vmla

namespace {

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s: far above any healthy pipeline wait
constexpr int kStages = 9;
constexpr int kMaxPos = 1024;  // RoPE range per axis [paperlayer App. C.1]

size_t esize(const vmla_config& c) { return c.dtype == VMLA_BF16 ? 2 : 4; }
int64_t tokens_per_frame(const vmla_config& c) { return (int64_t)c.grid_h * c.grid_w; }
int64_t ring_rows(const vmla_config& c) { return (int64_t)c.window_frames * tokens_per_frame(c); }
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct WsLayout {
  size_t kr_rot = 0, qt = 0, dq = 0, chunk = 0, obar = 0, recon = 0;  // offsets
  size_t base_bytes = 0;   // every design but RECON_ONCE
  size_t recon_bytes = 0;  // extra for RECON_ONCE
};

WsLayout ws_layout(const vmla_config& c) {
  const size_t e = esize(c);
  const size_t B = c.batch, nq = (size_t)c.chunk_frames * tokens_per_frame(c);
  const size_t dh = (size_t)c.d_nope + c.d_rope;
  WsLayout w;
  size_t off = 0;
  w.kr_rot = off;
  off = align256(off + B * ring_rows(c) * c.d_rope * e);
  w.qt = off;
  off = align256(off + B * c.n_heads * nq * (size_t)(c.d_latent + c.d_rope) * e);
  w.dq = off;
  off = align256(off + B * c.n_heads * nq * dh * e);
  w.chunk = off;  // a chunk's latents: [B][rows][d_c + d_rope] (plus a d_rope copy for fp32)
  off = align256(off + B * (size_t)c.window_frames * tokens_per_frame(c) * (size_t)(c.d_latent + 2 * c.d_rope) * e);
  w.obar = off;  // the folded output mixer's input: O_bar as a bf16 pair [2][B][rows][n_h * d_c]
  off = align256(off + (c.dtype == VMLA_BF16 ? 2 * B * nq * c.n_heads * (size_t)c.d_latent * 2 : 0));
  w.recon = off;
  w.base_bytes = off;
  w.recon_bytes = B * ring_rows(c) * 2 * (size_t)c.n_heads * c.d_value * e;
  return w;
}

// A forced append column split the shape can take: one MMA covers at most 256 columns.
bool append_tiling_fits(const vmla_config& c, int n_split) {
  if (n_split == 0) return true;
  return append_part_cols(c.d_latent + c.d_rope, n_split) <= 256;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Detail of the last VMLA_ERR_CUDA returned on this thread (vmla_last_error_detail).
thread_local char g_detail[160] = "";

vmla_status cuda_fail(cudaError_t e) {
  std::snprintf(g_detail, sizeof(g_detail), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return VMLA_ERR_CUDA;
}
vmla_status map_fail() {
  std::snprintf(g_detail, sizeof(g_detail), "cuTensorMapEncodeTiled refused a tensor map (or the driver entry point is missing)");
  return VMLA_ERR_CUDA;
}
vmla_status cuda_status(cudaError_t e) { return e == cudaSuccess ? VMLA_OK : cuda_fail(e); }

// AUTO keeps the design measured fastest on one B200 that also meets the accuracy gate (relative
// L2 <= 1e-2, max |err| <= 3e-2 RMS against the fp64 definition):
//  - d_latent >= 192, or a split the absorbed kernel does not hold (past 256 latent dims; 64 or 96
//    rotary dims past 192): RECON_ONCE.  Per (query, key, head) the per-head attention multiplies
//    2 d_head = 256 pairs where the absorbed one multiplies 2 d_latent + d_rope (416 at 192), and
//    rebuilding the window's per-head K/V costs about 2 us per 1000 keys (Wan-1.3B layer: 0.87 ms
//    against 1.05 ms per call).  Its per-head K, V, queries and probabilities are fp16, which keeps
//    it inside the gate on every window, the shortest (600 keys) included;
//  - d_latent 64 or 128: ABSORBED, whose extra MMA work is then no larger than the reconstruction's
//    (0.84 against 0.86 ms per call at d_latent 64, 0.87 against 0.87 at 128, Wan layer), and which
//    needs no per-head workspace.
vmla_design resolve_design(const vmla_config& c, vmla_design d, int64_t n_keys) {
  (void)n_keys;
  if (d != VMLA_DESIGN_AUTO) return d;
  if (c.dtype != VMLA_BF16) return VMLA_DESIGN_ABSORBED;
  if (!attn_absorbed_supported(c.d_latent, c.d_rope) || c.d_latent >= 192) return VMLA_DESIGN_RECON_ONCE;
  return VMLA_DESIGN_ABSORBED;
}

// Whether some call of this configuration may run RECON_ONCE (its workspace must hold the window's
// per-head K/V): the design AUTO takes on the largest window, or RECON_ONCE asked for.
bool may_run_recon_once(const vmla_config& c, vmla_design d) {
  const int64_t max_keys = (int64_t)c.window_frames * c.grid_h * c.grid_w;
  return resolve_design(c, d, max_keys) == VMLA_DESIGN_RECON_ONCE;
}

}  // namespace

// ---------------------------------------------------------------- handle
struct vmla_handle {
  vmla_config cfg;
  void* ckv = nullptr;
  void* kr = nullptr;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  void* dense = nullptr;
  std::vector<int64_t> frames;        // latent cache, per layer
  std::vector<int64_t> dense_frames;  // dense cache, per layer
  unsigned* err = nullptr;            // device status word (resolved at bind)
  int append_split = 0;               // append work split (0: chosen per call), see vmla_set_append_tiling
  int append_rows = 0;                // 128-row tiles per append work item (0 or 1: one; 2: two)
  int append_ctas = 0;
  bool profiling = false;
  struct Timer {
    std::vector<cudaEvent_t> ev;  // begin/end pairs
    size_t used = 0;
  } timers[kStages];
  // vmla_chunk_step_host: the input copies run on their own stream, each after the previous
  // call's last reader of its staging buffer (x: the append, q: the attention)
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t x_ready = nullptr, q_ready = nullptr, x_free = nullptr, q_free = nullptr;
  // ... and the output comes back on a second one, a group of heads at a time
  cudaStream_t out_stream = nullptr;
  cudaEvent_t out_group = nullptr, out_done = nullptr;
  // reconstruct-once: the per-head queries are prepared on a stream of the handle's own while the
  // reconstruction runs on the caller's
  cudaStream_t side_stream = nullptr;
  cudaEvent_t side_fork = nullptr, side_join = nullptr;
};

namespace {

struct StageScope {  // CUDA events around one stage's launch(es) when profiling
  vmla_handle* h;
  int stage;
  cudaStream_t s;
  bool on = false;
  StageScope(vmla_handle* h_, int st, cudaStream_t s_) : h(h_), stage(st), s(s_) {
    if (!h->profiling) return;
    auto& t = h->timers[stage];
    if (t.used + 2 > t.ev.size()) {
      for (int k = 0; k < 2; ++k) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return;
        t.ev.push_back(e);
      }
    }
    on = cudaEventRecord(t.ev[t.used], s) == cudaSuccess;
  }
  ~StageScope() {
    if (!on) return;
    auto& t = h->timers[stage];
    cudaEventRecord(t.ev[t.used + 1], s);
    t.used += 2;
  }
};

// The device status word of the current device, resolved at the first launch.
vmla_status ensure_err(vmla_handle* h) {
  if (!h->err) h->err = device_error_word();
  return h->err ? VMLA_OK : VMLA_ERR_CUDA;
}

vmla_status check_layer(const vmla_handle* h, int layer) {
  if (!h) return VMLA_ERR_INVALID_ARG;
  if (layer < 0 || layer >= h->cfg.layers) return VMLA_ERR_OUT_OF_RANGE;
  return VMLA_OK;
}

// Frame rule of an append: a new chunk right after the newest frame, or a
// rewrite of the newest frames (a further denoising pass).
vmla_status check_append_frames(const vmla_config& c, int64_t F, int64_t first, int n, int64_t* new_F) {
  // one append never wraps onto its own frames: at most the ring's local part
  if (n < 1 || n > c.window_frames - c.sink_frames) return VMLA_ERR_OUT_OF_RANGE;
  if (first < 0) return VMLA_ERR_STATE;
  if (first == F)
    *new_F = F + n;
  else if (first + n == F)
    *new_F = F;
  else
    return VMLA_ERR_STATE;
  return VMLA_OK;
}

vmla_status check_attention_frames(const vmla_config& c, int64_t F, int64_t first, int n, Window* w) {
  if (n < 1 || n > c.chunk_frames) return VMLA_ERR_OUT_OF_RANGE;
  if (F < 1 || first < 0 || first + n != F) return VMLA_ERR_STATE;
  *w = window_of(c, F);
  return VMLA_OK;
}

template <class T>
T* at(void* base, size_t byte_off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + byte_off);
}

size_t layer_cache_offset(const vmla_config& c, int layer, int width) {
  return (size_t)layer * c.batch * ring_rows(c) * width * esize(c);
}

}  // namespace

extern "C" {

const char* vmla_status_string(vmla_status s) {
  switch (s) {
    case VMLA_OK: return "VMLA_OK";
    case VMLA_ERR_INVALID_ARG: return "VMLA_ERR_INVALID_ARG";
    case VMLA_ERR_UNSUPPORTED_SHAPE: return "VMLA_ERR_UNSUPPORTED_SHAPE";
    case VMLA_ERR_OUT_OF_RANGE: return "VMLA_ERR_OUT_OF_RANGE";
    case VMLA_ERR_CUDA: return "VMLA_ERR_CUDA";
    case VMLA_ERR_DEVICE_TIMEOUT: return "VMLA_ERR_DEVICE_TIMEOUT";
    case VMLA_ERR_STATE: return "VMLA_ERR_STATE";
    case VMLA_ERR_DEVICE_BOUNDS: return "VMLA_ERR_DEVICE_BOUNDS";
    case VMLA_ERR_DEVICE_RANGE: return "VMLA_ERR_DEVICE_RANGE";
  }
  return "VMLA_ERR_UNKNOWN";
}

int vmla_abi_version(void) { return VMLA_ABI_VERSION; }

vmla_status vmla_config_init(vmla_config* c) {
  if (!c) return VMLA_ERR_INVALID_ARG;
  std::memset(c, 0, sizeof(*c));
  c->d_model = 1536;
  c->n_heads = 12;
  c->d_nope = 96;
  c->d_rope = 32;
  c->d_latent = 192;
  c->d_value = 128;
  c->rope_pairs[0] = 6;
  c->rope_pairs[1] = 5;
  c->rope_pairs[2] = 5;
  c->rope_theta = 10000.f;
  c->grid_h = 30;
  c->grid_w = 52;
  c->window_frames = 21;
  c->chunk_frames = 3;
  c->batch = 1;
  c->layers = 1;
  c->dtype = VMLA_BF16;
  c->rope_mode = VMLA_ROPE_AT_READ;
  c->softmax_rescale_log2 = 8.f;
  c->sink_frames = 0;
  return VMLA_OK;
}

vmla_status vmla_config_check(const vmla_config* c) {
  if (!c) return VMLA_ERR_INVALID_ARG;
  if (c->dtype != VMLA_BF16 && c->dtype != VMLA_FP32) return VMLA_ERR_INVALID_ARG;
  if (c->rope_mode != VMLA_ROPE_AT_READ && c->rope_mode != VMLA_ROPE_AT_APPEND) return VMLA_ERR_INVALID_ARG;
  if (c->d_model < 1 || c->n_heads < 1 || c->d_nope < 0 || c->d_rope < 0 || c->d_latent < 1 || c->d_value < 1 ||
      c->grid_h < 1 || c->grid_w < 1 || c->window_frames < 1 || c->chunk_frames < 1 || c->batch < 1 ||
      c->layers < 1 || !(c->rope_theta > 0.f) || !(c->softmax_rescale_log2 >= 0.f))
    return VMLA_ERR_INVALID_ARG;
  int pairs = 0;
  for (int a = 0; a < 3; ++a) {
    if (c->rope_pairs[a] < 0 || c->rope_base_dims[a] < 0) return VMLA_ERR_INVALID_ARG;
    pairs += c->rope_pairs[a];
  }
  if (2 * pairs != c->d_rope || pairs > kMaxPairs) return VMLA_ERR_INVALID_ARG;
  if (c->chunk_frames > c->window_frames) return VMLA_ERR_INVALID_ARG;
  // a sink needs room for a whole chunk beside it, and window-relative positions
  if (c->sink_frames < 0 || c->sink_frames + c->chunk_frames > c->window_frames) return VMLA_ERR_INVALID_ARG;
  if (c->sink_frames > 0 && c->rope_mode != VMLA_ROPE_AT_READ) return VMLA_ERR_INVALID_ARG;
  if (c->d_value != c->d_nope + c->d_rope) return VMLA_ERR_UNSUPPORTED_SHAPE;  // dense layout [2][n_h][d_head]
  if (c->grid_h >= kMaxPos || c->grid_w >= kMaxPos || c->window_frames >= kMaxPos) return VMLA_ERR_OUT_OF_RANGE;
  if (c->dtype == VMLA_BF16) {
    // d_head 128 split 96/32 with d_latent 64..512, or 112/16, 64/64, 32/96 with d_latent 64..256
    if (c->d_value != 128 || c->d_nope + c->d_rope != 128) return VMLA_ERR_UNSUPPORTED_SHAPE;
    if (!(c->d_latent == 64 || c->d_latent == 128 || c->d_latent == 192 || c->d_latent == 256 || c->d_latent == 384 ||
          c->d_latent == 512))
      return VMLA_ERR_UNSUPPORTED_SHAPE;
    if (c->d_rope != 32 && !((c->d_rope == 16 || c->d_rope == 64 || c->d_rope == 96) && c->d_latent <= 256))
      return VMLA_ERR_UNSUPPORTED_SHAPE;
    if (c->d_model % 64 != 0) return VMLA_ERR_UNSUPPORTED_SHAPE;
  } else {
    if (c->d_latent + c->d_rope > 1024 || c->d_value > 1024) return VMLA_ERR_UNSUPPORTED_SHAPE;
  }
  return VMLA_OK;
}

vmla_status vmla_cache_bytes(const vmla_config* c, size_t* ckv, size_t* kr, size_t* dense) {
  vmla_status st = vmla_config_check(c);
  if (st != VMLA_OK) return st;
  const size_t rows = (size_t)c->layers * c->batch * ring_rows(*c);
  if (ckv) *ckv = rows * c->d_latent * esize(*c);
  if (kr) *kr = rows * c->d_rope * esize(*c);
  if (dense) *dense = rows * 2 * (size_t)c->n_heads * c->d_value * esize(*c);
  return VMLA_OK;
}

vmla_status vmla_workspace_bytes(const vmla_config* c, vmla_design d, size_t* bytes) {
  vmla_status st = vmla_config_check(c);
  if (st != VMLA_OK) return st;
  if (!bytes || d < VMLA_DESIGN_AUTO || d > VMLA_DESIGN_RECON_ONCE) return VMLA_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(*c);
  *bytes = w.base_bytes + (may_run_recon_once(*c, d) ? w.recon_bytes : 0);
  return VMLA_OK;
}

vmla_status vmla_workspace_offsets(const vmla_config* c, size_t* offsets, int n) {
  vmla_status st = vmla_config_check(c);
  if (st != VMLA_OK) return st;
  if (!offsets || n < VMLA_WS_COUNT) return VMLA_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(*c);
  offsets[VMLA_WS_KR_ROT] = w.kr_rot;
  offsets[VMLA_WS_QT] = w.qt;
  offsets[VMLA_WS_QD] = w.dq;
  offsets[VMLA_WS_RECON] = w.recon;
  return VMLA_OK;
}

vmla_status vmla_rope_frequencies(const vmla_config* c, float* freqs, int n) {
  vmla_status st = vmla_config_check(c);
  if (st != VMLA_OK) return st;
  if (!freqs || n < c->d_rope / 2) return VMLA_ERR_INVALID_ARG;
  const Rope r = make_rope(*c);
  for (int p = 0; p < c->d_rope / 2; ++p) freqs[p] = r.freq[p];
  return VMLA_OK;
}

vmla_status vmla_create(const vmla_config* c, vmla_handle** out) {
  if (!out) return VMLA_ERR_INVALID_ARG;
  *out = nullptr;
  vmla_status st = vmla_config_check(c);
  if (st != VMLA_OK) return st;
  vmla_handle* h = new (std::nothrow) vmla_handle();
  if (!h) return VMLA_ERR_INVALID_ARG;
  h->cfg = *c;
  h->frames.assign(c->layers, 0);
  h->dense_frames.assign(c->layers, 0);
  *out = h;
  return VMLA_OK;
}

vmla_status vmla_destroy(vmla_handle* h) {
  if (!h) return VMLA_ERR_INVALID_ARG;
  for (auto& t : h->timers)
    for (cudaEvent_t e : t.ev) cudaEventDestroy(e);
  for (cudaEvent_t e : {h->x_ready, h->q_ready, h->x_free, h->q_free, h->out_group, h->out_done, h->side_fork,
                        h->side_join})
    if (e) cudaEventDestroy(e);
  if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
  if (h->out_stream) cudaStreamDestroy(h->out_stream);
  if (h->side_stream) cudaStreamDestroy(h->side_stream);
  delete h;
  return VMLA_OK;
}

vmla_status vmla_bind(vmla_handle* h, void* ckv, void* kr, void* ws, size_t ws_bytes) {
  if (!h || !ckv || !kr || !ws) return VMLA_ERR_INVALID_ARG;
  if (!aligned16(ckv) || !aligned16(kr) || !aligned16(ws)) return VMLA_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(h->cfg);
  if (ws_bytes < w.base_bytes) return VMLA_ERR_INVALID_ARG;
  h->ckv = ckv;
  h->kr = kr;
  h->ws = ws;
  h->ws_bytes = ws_bytes;
  h->frames.assign(h->cfg.layers, 0);
  return VMLA_OK;
}

vmla_status vmla_dense_bind(vmla_handle* h, void* dense) {
  if (!h || !dense || !aligned16(dense)) return VMLA_ERR_INVALID_ARG;
  // the dense layout stores keys rotated at absolute positions: no window-relative re-indexing
  if (h->cfg.sink_frames > 0) return VMLA_ERR_UNSUPPORTED_SHAPE;
  h->dense = dense;
  h->dense_frames.assign(h->cfg.layers, 0);
  return VMLA_OK;
}

vmla_status vmla_window(const vmla_handle* h, int64_t F, int32_t* frame, int32_t* slot, int32_t* t_local,
                        int capacity, int* n) {
  if (!h || !n || F < 0) return VMLA_ERR_INVALID_ARG;
  const vmla_config& c = h->cfg;
  const Ring g = make_ring(c);
  const Window w = window_of(c, F);
  const int sink = (int)std::min<int64_t>(c.sink_frames, F);
  const int count = sink + (int)(F - w.local_start);
  *n = count;
  if (count > capacity) return VMLA_ERR_INVALID_ARG;
  for (int k = 0; k < count; ++k) {  // sink frames, then local frames oldest first
    const int64_t f = k < sink ? k : w.local_start + (k - sink);
    const int sl = (int)ring_frame_slot(g, f);
    if (frame) frame[k] = (int32_t)f;
    if (slot) slot[k] = (int32_t)sl;
    // RoPE at read: t from the slot, by the same function the window-RoPE kernel applies to every key
    // it rotates; RoPE at append: the keys were rotated with their absolute frame index when written
    if (t_local)
      t_local[k] = c.rope_mode == VMLA_ROPE_AT_APPEND ? (int32_t)f : (int32_t)ring_slot_t(g, sl, w.start_slot);
  }
  return VMLA_OK;
}

vmla_status vmla_state_get(const vmla_handle* h, int layer, int64_t* F) {
  vmla_status st = check_layer(h, layer);
  if (st != VMLA_OK) return st;
  if (!F) return VMLA_ERR_INVALID_ARG;
  *F = h->frames[layer];
  return VMLA_OK;
}

vmla_status vmla_state_set(vmla_handle* h, int layer, int64_t F) {
  vmla_status st = check_layer(h, layer);
  if (st != VMLA_OK) return st;
  if (F < 0) return VMLA_ERR_INVALID_ARG;
  h->frames[layer] = F;
  return VMLA_OK;
}

namespace {
// Every host-side check of a cache append (no CUDA call); *new_F gets the layer's frame count after it.
vmla_status append_args(vmla_handle* h, int layer, const void* x, const void* w_down, int64_t first, int n,
                        int64_t* new_F) {
  vmla_status st = check_layer(h, layer);
  if (st != VMLA_OK) return st;
  if (!h->ckv) return VMLA_ERR_STATE;
  if (!x || !w_down || !aligned16(x) || !aligned16(w_down)) return VMLA_ERR_INVALID_ARG;
  const vmla_config& c = h->cfg;
  if ((st = check_append_frames(c, h->frames[layer], first, n, new_F)) != VMLA_OK) return st;
  if (c.rope_mode == VMLA_ROPE_AT_APPEND && first + n > kMaxPos) return VMLA_ERR_OUT_OF_RANGE;
  if (c.dtype == VMLA_BF16 && !append_tiling_fits(c, h->append_split)) return VMLA_ERR_UNSUPPORTED_SHAPE;
  return VMLA_OK;
}
}  // namespace

vmla_status vmla_cache_append(vmla_handle* h, int layer, const void* x, const void* w_down, int64_t first,
                              int n, void* stream) {
  int64_t new_F;
  vmla_status st = append_args(h, layer, x, w_down, first, n, &new_F);
  if (st != VMLA_OK || (st = ensure_err(h)) != VMLA_OK) return st;
  const vmla_config& c = h->cfg;
  const bool rotate = c.rope_mode == VMLA_ROPE_AT_APPEND;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rows = (int)(n * tokens_per_frame(c));
  cudaError_t e;
  {
    StageScope scope(h, 0, s);
    if (c.dtype == VMLA_FP32) {
      SimtAppend a;
      a.x = static_cast<const float*>(x);
      a.w_down = static_cast<const float*>(w_down);
      a.ckv = at<float>(h->ckv, layer_cache_offset(c, layer, c.d_latent));
      a.kr = at<float>(h->kr, layer_cache_offset(c, layer, c.d_rope));
      a.batch = c.batch;
      a.rows = rows;
      a.d_model = c.d_model;
      a.d_latent = c.d_latent;
      a.d_rope = c.d_rope;
      a.first_frame = first;
      a.rotate = rotate;
      a.contiguous = 0;
      a.out_rows = ring_rows(c);
      a.ring = make_ring(c);
      a.rope = make_rope(c);
      e = launch_append_simt(a, s);
    } else {
      CUtensorMap tx, tw;
      const int nout = c.d_latent + c.d_rope;
      const AppendPlan plan = append_tc_plan(nout, rows, c.batch, h->append_split, h->append_rows, h->append_ctas);
      const int parts = plan.parts;
      if (!map3(&tx, x, c.d_model, rows, c.batch, (uint64_t)c.d_model * 2, (uint64_t)rows * c.d_model * 2, 64, 128,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
          !map2(&tw, w_down, c.d_model, nout, (uint64_t)c.d_model * 2, 64, append_part_cols(nout, parts),
                CU_TENSOR_MAP_SWIZZLE_128B))
        return map_fail();
      AppendTc a;
      a.ckv = at<__nv_bfloat16>(h->ckv, layer_cache_offset(c, layer, c.d_latent));
      a.kr = at<__nv_bfloat16>(h->kr, layer_cache_offset(c, layer, c.d_rope));
      a.rows = rows;
      a.d_model = c.d_model;
      a.d_latent = c.d_latent;
      a.d_rope = c.d_rope;
      a.first_frame = first;
      a.rotate = rotate;
      a.contiguous = 0;
      a.ring_rows = ring_rows(c);
      a.ring = make_ring(c);
      a.rope = make_rope(c);
      a.err = h->err;
      a.limit_ns = kWaitLimitNs;
      e = launch_append_tc(tx, tw, a, c.batch, s, plan);
    }
  }
  if (e != cudaSuccess) return cuda_fail(e);
  h->frames[layer] = new_F;
  return VMLA_OK;
}

namespace {

vmla_status attention_fp32(vmla_handle* h, int layer, const void* q, const void* w_uk, const void* w_uv, void* out,
                           int64_t first, int n, const Window& win, cudaStream_t s) {
  const vmla_config& c = h->cfg;
  const WsLayout w = ws_layout(c);
  const bool at_read = c.rope_mode == VMLA_ROPE_AT_READ;
  float* kr_layer = at<float>(h->kr, layer_cache_offset(c, layer, c.d_rope));
  const float* kpos = kr_layer;
  cudaError_t e = cudaSuccess;
  if (at_read) {
    StageScope scope(h, 1, s);
    RopeWindow r{kr_layer, at<float>(h->ws, w.kr_rot), c.batch, win.n_keys, c.d_rope, win.start_slot,
                 make_ring(c), make_rope(c)};
    e = launch_rope_window_f32(r, s);
    kpos = at<float>(h->ws, w.kr_rot);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  const int nq = (int)(n * tokens_per_frame(c));
  {
    StageScope scope(h, 2, s);
    SimtQPrep a{static_cast<const float*>(q), static_cast<const float*>(w_uk), at<float>(h->ws, w.qt), c.batch, nq,
                c.n_heads, c.d_nope, c.d_rope, c.d_latent, 1, first - (at_read ? win.t_origin : 0), make_ring(c),
                make_rope(c)};
    e = launch_qprep_simt(a, s);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  {
    StageScope scope(h, 3, s);
    SimtAttn a;
    a.qt = at<float>(h->ws, w.qt);
    a.key = at<float>(h->ckv, layer_cache_offset(c, layer, c.d_latent));
    a.kpos = kpos;
    a.w_uv = static_cast<const float*>(w_uv);
    a.out = static_cast<float*>(out);
    a.batch = c.batch;
    a.n_q = nq;
    a.n_keys = win.n_keys;
    a.n_heads = c.n_heads;
    a.d_latent = c.d_latent;
    a.d_rope = c.d_rope;
    a.d_value = c.d_value;
    a.dense = 0;
    a.ring_rows = ring_rows(c);
    a.scale = 1.f / std::sqrt((float)(c.d_nope + c.d_rope));
    e = launch_attn_simt(a, s);
  }
  return cuda_status(e);
}

// Output rows wanted in host memory (vmla_chunk_step_host): the absorbed attention then runs as
// one launch per group of heads that fills the GPU once, and each group's columns are copied to
// the host on `stream` while the next group computes; `copied` tells the caller it was done.
struct HostOut {
  void* host;
  cudaStream_t stream;
  cudaEvent_t group, done;
  bool copied;
  cudaEvent_t q_read = nullptr;  // recorded once the query-prep kernel has read q (its last reader)
  bool q_recorded = false;
};

// Record hout->q_read right after the kernel that last reads q.
cudaError_t note_q_read(HostOut* hout, cudaStream_t s) {
  if (!hout || !hout->q_read) return cudaSuccess;
  cudaError_t e = cudaEventRecord(hout->q_read, s);
  hout->q_recorded = e == cudaSuccess;
  return e;
}

// Launch an attention kernel (grid y = heads) as one launch per group of heads that fills the GPU
// once, each group's output columns copied to the host on hout->stream while the next group
// computes; `stream` then waits for the last copy.  `launch` enqueues heads [a.h0, a.h0 + a.h_count).
extern "C++" template <class Launch>
cudaError_t launch_head_groups(const vmla_config& c, int nq, AttnTc a, const void* out, HostOut* hout,
                               cudaStream_t s, Launch launch) {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      sms = 148;
  }
  const int per_head = a.m_tiles * c.batch;  // CTAs of one head
  const int hg = std::max(1, std::min(c.n_heads, sms / std::max(1, per_head)));
  const size_t pitch = (size_t)c.n_heads * 128 * sizeof(float);
  cudaError_t e = cudaSuccess;
  for (int g0 = 0; g0 < c.n_heads && e == cudaSuccess; g0 += hg) {
    a.h0 = g0;
    a.h_count = std::min(hg, c.n_heads - g0);
    if ((e = launch(a)) != cudaSuccess || (e = cudaEventRecord(hout->group, s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(hout->stream, hout->group, 0)) != cudaSuccess)
      break;
    e = cudaMemcpy2DAsync(static_cast<char*>(hout->host) + (size_t)g0 * 128 * sizeof(float), pitch,
                          static_cast<const char*>(out) + (size_t)g0 * 128 * sizeof(float), pitch,
                          (size_t)a.h_count * 128 * sizeof(float), (size_t)c.batch * nq, cudaMemcpyDeviceToHost,
                          hout->stream);
  }
  if (e == cudaSuccess && (e = cudaEventRecord(hout->done, hout->stream)) == cudaSuccess)
    e = cudaStreamWaitEvent(s, hout->done, 0);
  hout->copied = e == cudaSuccess;
  return e;
}

vmla_status dense_q_launch(vmla_handle* h, const void* q, int nq, int64_t t_first, cudaStream_t s, bool f16,
                           HostOut* hout);
vmla_status dense_attention_bf16_launch(vmla_handle* h, const void* q_dev, const void* kv_base, void* out, int nq,
                                        int n_keys, int64_t t_first, int stage, cudaStream_t s, bool f16,
                                        HostOut* hout = nullptr, bool q_done = false);

// The folded output mixer: out = O_bar W_fold^T instead of the per-head W_uv,h.
struct FoldArgs {
  const void* w_fold;  // [d_out][n_h * d_c]
  int d_out;
};

// The absorbed query computed from the query latent: q~ = [A_h ; W_qr,h] c_Q.
struct QLatArgs {
  const void* c_q;     // [B][n_q][d_q]
  const void* w_qabs;  // [n_h][d_c + 32][d_q]
  int d_q;
};

vmla_status attention_bf16(vmla_handle* h, int layer, const void* q, const void* w_uk, const void* w_uv, void* out,
                           int64_t first, int n, const Window& win, vmla_design design, cudaStream_t s,
                           const FoldArgs* fold = nullptr, const QLatArgs* qlat = nullptr, HostOut* hout = nullptr) {
  const vmla_config& c = h->cfg;
  if (design == VMLA_DESIGN_RECONSTRUCT && !attn_reconstruct_supported(c.d_latent)) return VMLA_ERR_UNSUPPORTED_SHAPE;
  // rotary widths other than 32: every design but reconstruct-in-tile
  if (c.d_rope != 32 && design == VMLA_DESIGN_RECONSTRUCT) return VMLA_ERR_UNSUPPORTED_SHAPE;
  if (design == VMLA_DESIGN_ABSORBED && !attn_absorbed_supported(c.d_latent, c.d_rope)) return VMLA_ERR_UNSUPPORTED_SHAPE;
  const WsLayout w = ws_layout(c);
  const bool at_read = c.rope_mode == VMLA_ROPE_AT_READ;
  const int nq = (int)(n * tokens_per_frame(c));
  const int64_t t_first = first - (at_read ? win.t_origin : 0);
  __nv_bfloat16* ckv_layer = at<__nv_bfloat16>(h->ckv, layer_cache_offset(c, layer, c.d_latent));
  __nv_bfloat16* kr_layer = at<__nv_bfloat16>(h->kr, layer_cache_offset(c, layer, c.d_rope));
  // the window's positional keys, rotated with window-relative t into the workspace (bf16; the
  // cache's own values when rotated at append).  Reconstruct-once rotates them itself while it
  // rebuilds the per-head keys, so it takes the cache's keys as they are.
  const bool recon_once = design == VMLA_DESIGN_RECON_ONCE;
  const void* kpos = kr_layer;
  cudaError_t e = cudaSuccess;
  if (at_read && !recon_once) {
    StageScope scope(h, 1, s);
    RopeWindow r{kr_layer, at<char>(h->ws, w.kr_rot), c.batch, win.n_keys, c.d_rope, win.start_slot,
                 make_ring(c), make_rope(c)};
    e = launch_rope_window_bf16(r, s);
    kpos = at<char>(h->ws, w.kr_rot);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  const uint64_t rr = ring_rows(c);

  if (design == VMLA_DESIGN_RECON_ONCE) {
    if (h->ws_bytes < w.base_bytes + w.recon_bytes) return VMLA_ERR_STATE;
    __nv_bfloat16* recon = at<__nv_bfloat16>(h->ws, w.recon);
    // the per-head queries (independent of the reconstruction) on the handle's side stream, forked
    // from and joined back into `s`
    if (!h->side_stream) {
      if ((e = cudaStreamCreateWithFlags(&h->side_stream, cudaStreamNonBlocking)) != cudaSuccess) return cuda_fail(e);
      for (cudaEvent_t* ev : {&h->side_fork, &h->side_join})
        if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return cuda_fail(e);
    }
    if ((e = cudaEventRecord(h->side_fork, s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(h->side_stream, h->side_fork, 0)) != cudaSuccess)
      return cuda_fail(e);
    vmla_status qs = dense_q_launch(h, q, nq, t_first, h->side_stream, true, hout);
    if (qs != VMLA_OK) return qs;
    if ((e = cudaEventRecord(h->side_join, h->side_stream)) != cudaSuccess) return cuda_fail(e);
    {
      StageScope scope(h, 7, s);
      CUtensorMap tc, tuk, tuv;
      if (!map3(&tc, ckv_layer, c.d_latent, win.n_keys, c.batch, (uint64_t)c.d_latent * 2, rr * c.d_latent * 2, 64,
                128, CU_TENSOR_MAP_SWIZZLE_128B) ||
          !map3(&tuk, w_uk, c.d_latent, c.d_nope, c.n_heads, (uint64_t)c.d_latent * 2,
                (uint64_t)c.d_nope * c.d_latent * 2, 64, c.d_nope,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
          !map3(&tuv, w_uv, c.d_latent, 128, c.n_heads, (uint64_t)c.d_latent * 2, 128ull * c.d_latent * 2, 64, 128,
                CU_TENSOR_MAP_SWIZZLE_128B))
        return map_fail();
      ReconTc a;
      a.kr = kpos;
      a.dense = recon;
      a.f16 = 1;  // the window's per-head K/V in fp16: 2^-11 rounding per entry, past bf16's 2^-8
      a.rows = win.n_keys;
      a.n_heads = c.n_heads;
      a.d_latent = c.d_latent;
      a.d_rope = c.d_rope;
      a.first_frame = 0;
      a.rotate = 0;
      a.window_t = at_read;  // rotated here with window-relative t (or already at append)
      a.window_start_slot = win.start_slot;
      a.to_ring = 0;
      a.kr_rows = rr;
      a.kr_stride = c.d_rope;
      a.ring_rows = rr;
      a.ring = make_ring(c);
      a.rope = make_rope(c);
      a.err = h->err;
      a.limit_ns = kWaitLimitNs;
      CUtensorMap to;
      const uint64_t row_bytes = 2ull * c.n_heads * 128 * 2;
      if (!map3(&to, recon, 2ull * c.n_heads * 128, win.n_keys, c.batch, row_bytes, rr * row_bytes, 64, 128,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
        return map_fail();
      e = launch_recon_tc(tc, tuk, tuv, &to, a, c.batch, s);
    }
    if (e != cudaSuccess || (e = cudaStreamWaitEvent(s, h->side_join, 0)) != cudaSuccess) return cuda_fail(e);
    return dense_attention_bf16_launch(h, q, recon, out, nq, win.n_keys, t_first, 6, s, true, hout, true);
  }
  if (design == VMLA_DESIGN_RECONSTRUCT) {
    __nv_bfloat16* qd = at<__nv_bfloat16>(h->ws, w.dq);
    {
      StageScope scope(h, 2, s);
      DenseQTc a{static_cast<const __nv_bfloat16*>(q), qd, c.batch, nq, c.n_heads, c.d_rope, t_first, make_ring(c),
                 make_rope(c)};
      e = launch_dense_q_bf16(a, s);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    StageScope scope(h, 4, s);
    CUtensorMap tq, tc, tkr, tuk, tuv, to;
    if (!map3(&tq, qd, 128, nq, (uint64_t)c.batch * c.n_heads, 256, (uint64_t)nq * 256, 64, 128,
              CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map3(&tc, ckv_layer, c.d_latent, win.n_keys, c.batch, (uint64_t)c.d_latent * 2, rr * c.d_latent * 2, 64, 128,
              CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map3(&tkr, kpos, 32, win.n_keys, c.batch, 64, rr * 64, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !map3(&tuk, w_uk, c.d_latent, c.d_nope, c.n_heads, (uint64_t)c.d_latent * 2,
              (uint64_t)c.d_nope * c.d_latent * 2, 64, c.d_nope,
              CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map3(&tuv, w_uv, c.d_latent, 128, c.n_heads, (uint64_t)c.d_latent * 2, 128ull * c.d_latent * 2, 64, 128,
              CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map3(&to, out, (uint64_t)c.n_heads * 128, nq, c.batch, (uint64_t)c.n_heads * 128 * 4,
              (uint64_t)nq * c.n_heads * 128 * 4, 32, 128, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_DATA_TYPE_FLOAT32))
      return map_fail();
    AttnTc a;
    a.n_q = nq;
    a.n_keys = win.n_keys;
    a.n_heads = c.n_heads;
    a.m_tiles = (nq + 127) / 128;
    a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)(c.d_nope + c.d_rope)));
    a.rescale_threshold = c.softmax_rescale_log2;
    a.err = h->err;
    a.limit_ns = kWaitLimitNs;
    return cuda_status(launch_attn_reconstruct_tc(c.d_latent, tq, tc, tkr, tuk, tuv, to, a, c.batch, s));
  }

  __nv_bfloat16* qt = at<__nv_bfloat16>(h->ws, w.qt);
  const int dqk = c.d_latent + c.d_rope;
  if (qlat) {
    StageScope scope(h, 2, s);
    CUtensorMap tcq, tw, tqt;
    if (!map3(&tcq, qlat->c_q, qlat->d_q, nq, c.batch, (uint64_t)qlat->d_q * 2, (uint64_t)nq * qlat->d_q * 2, 64, 128,
              CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map3(&tw, qlat->w_qabs, qlat->d_q, dqk, c.n_heads, (uint64_t)qlat->d_q * 2, (uint64_t)dqk * qlat->d_q * 2, 64,
              dqk, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map3(&tqt, qt, dqk, nq, (uint64_t)c.batch * c.n_heads, (uint64_t)dqk * 2, (uint64_t)nq * dqk * 2, 64, 64,
              CU_TENSOR_MAP_SWIZZLE_128B))
      return map_fail();
    QLatTc a;
    a.qt = qt;
    a.n_q = nq;
    a.n_heads = c.n_heads;
    a.d_latent = c.d_latent;
    a.d_rope = c.d_rope;
    a.d_q = qlat->d_q;
    a.t_first = t_first;
    a.ring = make_ring(c);
    a.rope = make_rope(c);
    a.err = h->err;
    a.limit_ns = kWaitLimitNs;
    e = launch_qlat_tc(tcq, tw, tqt, a, c.batch, s);
  } else {
    StageScope scope(h, 2, s);
    CUtensorMap tq, tuk, tqt;
    if (!map3(&tq, q, (uint64_t)c.n_heads * 128, nq, c.batch, (uint64_t)c.n_heads * 128 * 2,
              (uint64_t)nq * c.n_heads * 128 * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map3(&tuk, w_uk, c.d_latent, c.d_nope, c.n_heads, (uint64_t)c.d_latent * 2,
              (uint64_t)c.d_nope * c.d_latent * 2, 64, c.d_nope, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map3(&tqt, qt, dqk, nq, (uint64_t)c.batch * c.n_heads, (uint64_t)dqk * 2, (uint64_t)nq * dqk * 2, 64, 64,
              CU_TENSOR_MAP_SWIZZLE_128B))
      return map_fail();
    QPrepTc a;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.qt = qt;
    a.n_q = nq;
    a.n_heads = c.n_heads;
    a.d_latent = c.d_latent;
    a.d_rope = c.d_rope;
    a.t_first = t_first;
    a.ring = make_ring(c);
    a.rope = make_rope(c);
    a.err = h->err;
    a.limit_ns = kWaitLimitNs;
    e = launch_qprep_tc(tq, tuk, tqt, a, c.batch, s);
  }
  if (e == cudaSuccess) e = note_q_read(hout, s);
  if (e != cudaSuccess) return cuda_fail(e);
  {
    StageScope scope(h, 3, s);
    const int bn = attn_absorbed_block_n(c.d_latent);
    const uint64_t bh = (uint64_t)c.batch * c.n_heads;
    CUtensorMap tq, tqr, tk, tkr, tuv, to;
    // the rotary columns: one box c.d_rope wide, swizzled at its row width (32, 64 or 128 bytes)
    // (96 rotary dims: three boxes of 32, 64-byte swizzle)
    const int rbox = c.d_rope == 96 ? 32 : c.d_rope;
    const CUtensorMapSwizzle rsw = rbox == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                              : (rbox == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    const uint64_t rb = (uint64_t)c.d_rope * 2;
    if (!map3(&tq, qt, dqk, nq, bh, (uint64_t)dqk * 2, (uint64_t)nq * dqk * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map3(&tqr, qt, dqk, nq, bh, (uint64_t)dqk * 2, (uint64_t)nq * dqk * 2, rbox, 128, rsw) ||
        !map3(&tk, ckv_layer, c.d_latent, win.n_keys, c.batch, (uint64_t)c.d_latent * 2, rr * c.d_latent * 2, 64, bn,
              CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map3(&tkr, kpos, c.d_rope, win.n_keys, c.batch, rb, rr * rb, rbox, bn, rsw))
      return map_fail();
    if (!fold &&
        (!map3(&tuv, w_uv, c.d_latent, 128, c.n_heads, (uint64_t)c.d_latent * 2, 128ull * c.d_latent * 2, 64, 128,
               CU_TENSOR_MAP_SWIZZLE_128B) ||
         !map3(&to, out, (uint64_t)c.n_heads * 128, nq, c.batch, (uint64_t)c.n_heads * 128 * 4,
               (uint64_t)nq * c.n_heads * 128 * 4, 32, 128, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_DATA_TYPE_FLOAT32)))
      return map_fail();
    AttnTc a;
    a.n_q = nq;
    a.n_keys = win.n_keys;
    a.n_heads = c.n_heads;
    a.m_tiles = (nq + 127) / 128;
    a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)(c.d_nope + c.d_rope)));
    a.rescale_threshold = c.softmax_rescale_log2;
    a.err = h->err;
    a.limit_ns = kWaitLimitNs;
    if (!fold && !hout) {
      e = launch_attn_absorbed_tc(c.d_latent, c.d_rope, tq, tqr, tk, tkr, tuv, to, a, c.batch, s);
    } else if (!fold) {
      e = launch_head_groups(c, nq, a, out, hout, s, [&](const AttnTc& ag) {
        return launch_attn_absorbed_tc(c.d_latent, c.d_rope, tq, tqr, tk, tkr, tuv, to, ag, c.batch, s);
      });
    } else {
      const uint64_t kf = (uint64_t)c.n_heads * c.d_latent;
      __nv_bfloat16* ob_hi = at<__nv_bfloat16>(h->ws, w.obar);
      __nv_bfloat16* ob_lo = ob_hi + (size_t)c.batch * nq * kf;
      CUtensorMap thi, tlo;
      if (!map3(&thi, ob_hi, kf, nq, c.batch, kf * 2, (uint64_t)nq * kf * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
          !map3(&tlo, ob_lo, kf, nq, c.batch, kf * 2, (uint64_t)nq * kf * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return map_fail();
      e = launch_attn_absorbed_obar_tc(c.d_latent, c.d_rope, tq, tqr, tk, tkr, thi, tlo, a, c.batch, s);
    }
  }
  if (e != cudaSuccess || !fold) return cuda_status(e);
  StageScope scope(h, 8, s);
  const uint64_t kf = (uint64_t)c.n_heads * c.d_latent, rows = (uint64_t)c.batch * nq;
  __nv_bfloat16* ob_hi = at<__nv_bfloat16>(h->ws, w.obar);
  __nv_bfloat16* ob_lo = ob_hi + rows * kf;
  CUtensorMap thi, tlo, tw, to;
  if (!map3(&thi, ob_hi, kf, rows, 1, kf * 2, rows * kf * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map3(&tlo, ob_lo, kf, rows, 1, kf * 2, rows * kf * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map3(&tw, fold->w_fold, kf, fold->d_out, 1, kf * 2, (uint64_t)fold->d_out * kf * 2, 64, 128,
            CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map3(&to, out, fold->d_out, rows, 1, (uint64_t)fold->d_out * 4, rows * fold->d_out * 4, 32, 128,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_FLOAT32))
    return map_fail();
  FoldTc fa{(int)rows, (int)kf, fold->d_out, h->err, kWaitLimitNs};
  return cuda_status(launch_fold_gemm_tc(thi, tlo, tw, to, fa, s));
}

// Dense d_head = 128 attention on a per-head K/V buffer [B][ring_rows][2][n_h][128]: bf16 (the
// dense cache) or, with f16, fp16 (the reconstruct-once workspace; the queries then go fp16 too).
// The per-head queries [B][n_h][n_q][128] in the workspace: q_nope copied, q_rope rotated.
vmla_status dense_q_launch(vmla_handle* h, const void* q, int nq, int64_t t_first, cudaStream_t s, bool f16,
                           HostOut* hout) {
  const vmla_config& c = h->cfg;
  const WsLayout w = ws_layout(c);
  cudaError_t e;
  {
    StageScope scope(h, 2, s);
    DenseQTc a{static_cast<const __nv_bfloat16*>(q), at<char>(h->ws, w.dq), c.batch, nq, c.n_heads, c.d_rope,
               t_first, make_ring(c), make_rope(c)};
    a.f16 = f16;
    a.err = h->err;
    e = launch_dense_q_bf16(a, s);
  }
  if (e == cudaSuccess) e = note_q_read(hout, s);
  return e == cudaSuccess ? VMLA_OK : cuda_fail(e);
}

vmla_status dense_attention_bf16_launch(vmla_handle* h, const void* q, const void* kv_base, void* out, int nq,
                                        int n_keys, int64_t t_first, int stage, cudaStream_t s, bool f16,
                                        HostOut* hout, bool q_done) {
  const vmla_config& c = h->cfg;
  const WsLayout w = ws_layout(c);
  void* qd = at<char>(h->ws, w.dq);
  vmla_status st;
  if (!q_done && (st = dense_q_launch(h, q, nq, t_first, s, f16, hout)) != VMLA_OK) return st;
  StageScope scope(h, stage, s);
  const uint64_t rr = ring_rows(c);
  const uint64_t row_bytes = 2ull * c.n_heads * 128 * 2;
  CUtensorMap tq, tkv, to;
  const CUtensorMapDataType et = f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!map3(&tq, qd, 128, nq, (uint64_t)c.batch * c.n_heads, 256, (uint64_t)nq * 256, 64, 128,
            CU_TENSOR_MAP_SWIZZLE_128B, et) ||
      !map3(&tkv, kv_base, 2ull * c.n_heads * 128, n_keys, c.batch, row_bytes, rr * row_bytes, 64,
            attn_dense_block_n(), CU_TENSOR_MAP_SWIZZLE_128B, et) ||
      !map3(&to, out, (uint64_t)c.n_heads * 128, nq, c.batch, (uint64_t)c.n_heads * 128 * 4,
            (uint64_t)nq * c.n_heads * 128 * 4, 32, 128, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_FLOAT32))
    return map_fail();
  AttnTc a;
  a.n_q = nq;
  a.n_keys = n_keys;
  a.n_heads = c.n_heads;
  a.m_tiles = (nq + 127) / 128;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)(c.d_nope + c.d_rope)));
  a.rescale_threshold = c.softmax_rescale_log2;
  a.err = h->err;
  a.limit_ns = kWaitLimitNs;
  if (hout)
    return cuda_status(launch_head_groups(c, nq, a, out, hout, s, [&](const AttnTc& ag) {
      return launch_attn_dense_tc(tq, tkv, to, ag, c.batch, s, f16);
    }));
  return cuda_status(launch_attn_dense_tc(tq, tkv, to, a, c.batch, s, f16));
}

}  // namespace

namespace {
// Every host-side check of a chunk attention call (no CUDA call) when the layer holds `frames`
// frames; *design gets the design that runs and *win the window.
vmla_status attention_args(vmla_handle* h, int layer, const void* q, const void* w_uk, const void* w_uv,
                           const void* out, int64_t first, int n, vmla_design* design, int64_t frames, Window* win) {
  vmla_status st = check_layer(h, layer);
  if (st != VMLA_OK) return st;
  if (!h->ckv) return VMLA_ERR_STATE;
  if (!q || !w_uk || !w_uv || !out || !aligned16(q) || !aligned16(w_uk) || !aligned16(w_uv) || !aligned16(out))
    return VMLA_ERR_INVALID_ARG;
  if (*design < VMLA_DESIGN_AUTO || *design > VMLA_DESIGN_RECON_ONCE) return VMLA_ERR_INVALID_ARG;
  const vmla_config& c = h->cfg;
  if ((st = check_attention_frames(c, frames, first, n, win)) != VMLA_OK) return st;
  if (c.rope_mode == VMLA_ROPE_AT_APPEND && first + n > kMaxPos) return VMLA_ERR_OUT_OF_RANGE;
  const bool automatic = *design == VMLA_DESIGN_AUTO;
  *design = resolve_design(c, *design, win->n_keys);
  if (automatic && *design == VMLA_DESIGN_RECON_ONCE && c.d_latent <= 256 &&
      h->ws_bytes < ws_layout(c).base_bytes + ws_layout(c).recon_bytes)
    *design = VMLA_DESIGN_ABSORBED;  // AUTO with a workspace bound without room for the per-head K/V
  if (c.dtype == VMLA_BF16) {
    // the absorbed kernels keep d_latent + d_rope query and key columns resident: up to 256 latent dims
    if (*design == VMLA_DESIGN_ABSORBED && c.d_latent > 256) return VMLA_ERR_UNSUPPORTED_SHAPE;
    if (*design == VMLA_DESIGN_RECONSTRUCT && !attn_reconstruct_supported(c.d_latent))
      return VMLA_ERR_UNSUPPORTED_SHAPE;
    if (*design == VMLA_DESIGN_ABSORBED && !attn_absorbed_supported(c.d_latent, c.d_rope))
      return VMLA_ERR_UNSUPPORTED_SHAPE;
    if (c.d_rope != 32 && *design == VMLA_DESIGN_RECONSTRUCT) return VMLA_ERR_UNSUPPORTED_SHAPE;
    if (*design == VMLA_DESIGN_RECON_ONCE) {
      const WsLayout w = ws_layout(c);
      if (h->ws_bytes < w.base_bytes + w.recon_bytes) return VMLA_ERR_STATE;
    }
  }
  return VMLA_OK;
}

vmla_status chunk_attention(vmla_handle* h, int layer, const void* q, const void* w_uk, const void* w_uv, void* out,
                            int64_t first, int n, vmla_design design, void* stream, HostOut* hout) {
  Window win;
  vmla_status st = attention_args(h, layer, q, w_uk, w_uv, out, first, n, &design, h->frames[layer], &win);
  if (st != VMLA_OK || (st = ensure_err(h)) != VMLA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (h->cfg.dtype == VMLA_FP32) return attention_fp32(h, layer, q, w_uk, w_uv, out, first, n, win, s);
  return attention_bf16(h, layer, q, w_uk, w_uv, out, first, n, win, design, s, nullptr, nullptr,
                        design == VMLA_DESIGN_ABSORBED || design == VMLA_DESIGN_RECON_ONCE ? hout : nullptr);
}
}  // namespace

vmla_status vmla_chunk_attention(vmla_handle* h, int layer, const void* q, const void* w_uk, const void* w_uv,
                                 void* out, int64_t first, int n, vmla_design design, void* stream) {
  return chunk_attention(h, layer, q, w_uk, w_uv, out, first, n, design, stream, nullptr);
}

vmla_status vmla_fold_query_weights(const vmla_config* cfg, const void* w_uq, const void* w_qr, const void* w_uk,
                                    int d_q, void* w_qabs, void* stream) {
  if (!cfg || !w_uq || !w_qr || !w_uk || !w_qabs) return VMLA_ERR_INVALID_ARG;
  vmla_status st = vmla_config_check(cfg);
  if (st != VMLA_OK) return st;
  if (cfg->dtype != VMLA_BF16 || !qlat_supported(cfg->d_latent, cfg->d_rope, d_q))
    return VMLA_ERR_UNSUPPORTED_SHAPE;
  return cuda_status(launch_fold_query(static_cast<const __nv_bfloat16*>(w_uq), static_cast<const __nv_bfloat16*>(w_qr),
                                       static_cast<const __nv_bfloat16*>(w_uk), static_cast<__nv_bfloat16*>(w_qabs),
                                       cfg->n_heads, cfg->d_nope, cfg->d_rope, cfg->d_latent, d_q,
                                       static_cast<cudaStream_t>(stream)));
}

vmla_status vmla_chunk_attention_qlatent(vmla_handle* h, int layer, const void* c_q, const void* w_qabs, int d_q,
                                         const void* w_uv, void* out, int64_t first, int n, void* stream) {
  vmla_status st = check_layer(h, layer);
  if (st != VMLA_OK) return st;
  if (!h->ckv) return VMLA_ERR_STATE;
  if (!c_q || !w_qabs || !w_uv || !out || !aligned16(c_q) || !aligned16(w_qabs) || !aligned16(w_uv) ||
      !aligned16(out))
    return VMLA_ERR_INVALID_ARG;
  const vmla_config& c = h->cfg;
  if (c.dtype != VMLA_BF16 || !qlat_supported(c.d_latent, c.d_rope, d_q) || !attn_absorbed_supported(c.d_latent, c.d_rope))
    return VMLA_ERR_UNSUPPORTED_SHAPE;
  Window win;
  if ((st = check_attention_frames(c, h->frames[layer], first, n, &win)) != VMLA_OK) return st;
  if (c.rope_mode == VMLA_ROPE_AT_APPEND && first + n > kMaxPos) return VMLA_ERR_OUT_OF_RANGE;
  if ((st = ensure_err(h)) != VMLA_OK) return st;
  const QLatArgs ql{c_q, w_qabs, d_q};
  return attention_bf16(h, layer, nullptr, nullptr, w_uv, out, first, n, win, VMLA_DESIGN_ABSORBED,
                        static_cast<cudaStream_t>(stream), nullptr, &ql);
}

vmla_status vmla_fold_output_weights(const vmla_config* cfg, const void* w_o, const void* w_uv, void* w_fold,
                                     int d_out, void* stream) {
  if (!cfg || !w_o || !w_uv || !w_fold) return VMLA_ERR_INVALID_ARG;
  vmla_status st = vmla_config_check(cfg);
  if (st != VMLA_OK) return st;
  if (cfg->dtype != VMLA_BF16) return VMLA_ERR_UNSUPPORTED_SHAPE;
  if (d_out < 1) return VMLA_ERR_INVALID_ARG;
  return cuda_status(launch_fold_weights(static_cast<const __nv_bfloat16*>(w_o),
                                         static_cast<const __nv_bfloat16*>(w_uv), static_cast<__nv_bfloat16*>(w_fold),
                                         d_out, cfg->n_heads, cfg->d_value, cfg->d_latent,
                                         static_cast<cudaStream_t>(stream)));
}

vmla_status vmla_chunk_attention_folded(vmla_handle* h, int layer, const void* q, const void* w_uk,
                                        const void* w_fold, int d_out, void* out, int64_t first, int n,
                                        void* stream) {
  vmla_status st = check_layer(h, layer);
  if (st != VMLA_OK) return st;
  if (!h->ckv) return VMLA_ERR_STATE;
  if (!q || !w_uk || !w_fold || !out || !aligned16(q) || !aligned16(w_uk) || !aligned16(w_fold) || !aligned16(out))
    return VMLA_ERR_INVALID_ARG;
  const vmla_config& c = h->cfg;
  if (c.dtype != VMLA_BF16 || !attn_absorbed_supported(c.d_latent, c.d_rope) || d_out < 128 || d_out % 128 != 0)
    return VMLA_ERR_UNSUPPORTED_SHAPE;
  Window win;
  if ((st = check_attention_frames(c, h->frames[layer], first, n, &win)) != VMLA_OK) return st;
  if (c.rope_mode == VMLA_ROPE_AT_APPEND && first + n > kMaxPos) return VMLA_ERR_OUT_OF_RANGE;
  if ((st = ensure_err(h)) != VMLA_OK) return st;
  const FoldArgs fold{w_fold, d_out};
  return attention_bf16(h, layer, q, w_uk, nullptr, out, first, n, win, VMLA_DESIGN_ABSORBED,
                        static_cast<cudaStream_t>(stream), &fold);
}

vmla_status vmla_dense_cache_append(vmla_handle* h, int layer, const void* x, const void* w_down, const void* w_uk,
                                    const void* w_uv, int64_t first, int n, void* stream) {
  vmla_status st = check_layer(h, layer);
  if (st != VMLA_OK) return st;
  if (!h->dense || !h->ws) return VMLA_ERR_STATE;
  if (!x || !w_down || !w_uk || !w_uv || !aligned16(x) || !aligned16(w_down) || !aligned16(w_uk) || !aligned16(w_uv))
    return VMLA_ERR_INVALID_ARG;
  const vmla_config& c = h->cfg;
  int64_t new_F;
  if ((st = check_append_frames(c, h->dense_frames[layer], first, n, &new_F)) != VMLA_OK) return st;
  if (first + n > kMaxPos) return VMLA_ERR_OUT_OF_RANGE;
  if (c.dtype == VMLA_BF16 && !append_tiling_fits(c, h->append_split)) return VMLA_ERR_UNSUPPORTED_SHAPE;
  if ((st = ensure_err(h)) != VMLA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const WsLayout w = ws_layout(c);
  const int rows = (int)(n * tokens_per_frame(c));
  const size_t dense_off = (size_t)layer * c.batch * ring_rows(c) * 2 * c.n_heads * c.d_value * esize(c);
  cudaError_t e;
  StageScope scope(h, 5, s);
  if (c.dtype == VMLA_FP32) {
    float* cbuf = at<float>(h->ws, w.chunk);
    float* rbuf = cbuf + (size_t)c.batch * rows * c.d_latent;
    SimtAppend a;
    a.x = static_cast<const float*>(x);
    a.w_down = static_cast<const float*>(w_down);
    a.ckv = cbuf;
    a.kr = rbuf;
    a.batch = c.batch;
    a.rows = rows;
    a.d_model = c.d_model;
    a.d_latent = c.d_latent;
    a.d_rope = c.d_rope;
    a.first_frame = first;
    a.rotate = 0;
    a.contiguous = 1;
    a.out_rows = rows;
    a.ring = make_ring(c);
    a.rope = make_rope(c);
    if ((e = launch_append_simt(a, s)) != cudaSuccess) return cuda_fail(e);
    SimtDenseReconstruct d{cbuf, rbuf, static_cast<const float*>(w_uk), static_cast<const float*>(w_uv),
                           at<float>(h->dense, dense_off), c.batch, rows, c.n_heads, c.d_nope, c.d_rope,
                           c.d_latent, c.d_value, first, make_ring(c), make_rope(c)};
    e = launch_dense_reconstruct_simt(d, s);
  } else {
    __nv_bfloat16* chunk = at<__nv_bfloat16>(h->ws, w.chunk);  // [B][rows][d_c + 32]
    const int nout = c.d_latent + c.d_rope;
    const AppendPlan plan = append_tc_plan(nout, rows, c.batch, h->append_split, h->append_rows, h->append_ctas);
    const int parts = plan.parts;
    CUtensorMap tx, tw;
    if (!map3(&tx, x, c.d_model, rows, c.batch, (uint64_t)c.d_model * 2, (uint64_t)rows * c.d_model * 2, 64, 128,
              CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map2(&tw, w_down, c.d_model, nout, (uint64_t)c.d_model * 2, 64, append_part_cols(nout, parts),
              CU_TENSOR_MAP_SWIZZLE_128B))
      return map_fail();
    AppendTc a;
    a.ckv = chunk;
    a.kr = nullptr;
    a.rows = rows;
    a.d_model = c.d_model;
    a.d_latent = c.d_latent;
    a.d_rope = c.d_rope;
    a.first_frame = first;
    a.rotate = 0;
    a.contiguous = 1;
    a.ring_rows = rows;
    a.ring = make_ring(c);
    a.rope = make_rope(c);
    a.err = h->err;
    a.limit_ns = kWaitLimitNs;
    if ((e = launch_append_tc(tx, tw, a, c.batch, s, plan)) != cudaSuccess) return cuda_fail(e);
    CUtensorMap tc, tuk, tuv;
    if (!map3(&tc, chunk, c.d_latent, rows, c.batch, (uint64_t)nout * 2, (uint64_t)rows * nout * 2, 64, 128,
              CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map3(&tuk, w_uk, c.d_latent, c.d_nope, c.n_heads, (uint64_t)c.d_latent * 2,
              (uint64_t)c.d_nope * c.d_latent * 2, 64, c.d_nope,
              CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map3(&tuv, w_uv, c.d_latent, 128, c.n_heads, (uint64_t)c.d_latent * 2, 128ull * c.d_latent * 2, 64, 128,
              CU_TENSOR_MAP_SWIZZLE_128B))
      return map_fail();
    ReconTc r;
    r.f16 = 0;  // the dense comparison caches bf16 entries
    r.kr = chunk + c.d_latent;  // positional key columns of the chunk rows (row stride d_c + 32)
    r.dense = at<__nv_bfloat16>(h->dense, dense_off);
    r.rows = rows;
    r.n_heads = c.n_heads;
    r.d_latent = c.d_latent;
    r.d_rope = c.d_rope;
    r.first_frame = first;
    r.rotate = 1;
    r.to_ring = 1;
    r.kr_rows = rows;
    r.kr_stride = nout;
    r.ring_rows = ring_rows(c);
    r.ring = make_ring(c);
    r.rope = make_rope(c);
    r.err = h->err;
    r.limit_ns = kWaitLimitNs;
    e = launch_recon_tc(tc, tuk, tuv, nullptr, r, c.batch, s);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  h->dense_frames[layer] = new_F;
  return VMLA_OK;
}

vmla_status vmla_dense_chunk_attention(vmla_handle* h, int layer, const void* q, void* out, int64_t first, int n,
                                       void* stream) {
  vmla_status st = check_layer(h, layer);
  if (st != VMLA_OK) return st;
  if (!h->dense || !h->ws) return VMLA_ERR_STATE;
  if (!q || !out || !aligned16(q) || !aligned16(out)) return VMLA_ERR_INVALID_ARG;
  const vmla_config& c = h->cfg;
  Window win;
  if ((st = check_attention_frames(c, h->dense_frames[layer], first, n, &win)) != VMLA_OK) return st;
  if (first + n > kMaxPos) return VMLA_ERR_OUT_OF_RANGE;
  if ((st = ensure_err(h)) != VMLA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const WsLayout w = ws_layout(c);
  const int nq = (int)(n * tokens_per_frame(c));
  const size_t dense_off = (size_t)layer * c.batch * ring_rows(c) * 2 * c.n_heads * c.d_value * esize(c);
  if (c.dtype == VMLA_BF16)
    return dense_attention_bf16_launch(h, q, at<char>(h->dense, dense_off), out, nq, win.n_keys, first, 6, s, false);
  cudaError_t e;
  {
    StageScope scope(h, 2, s);
    SimtQPrep a{static_cast<const float*>(q), nullptr, at<float>(h->ws, w.dq), c.batch, nq, c.n_heads, c.d_nope,
                c.d_rope, c.d_latent, 0, first, make_ring(c), make_rope(c)};
    if ((e = launch_qprep_simt(a, s)) != cudaSuccess) return cuda_fail(e);
  }
  StageScope scope(h, 6, s);
  SimtAttn a;
  a.qt = at<float>(h->ws, w.dq);
  a.key = at<float>(h->dense, dense_off);
  a.kpos = nullptr;
  a.w_uv = nullptr;
  a.out = static_cast<float*>(out);
  a.batch = c.batch;
  a.n_q = nq;
  a.n_keys = win.n_keys;
  a.n_heads = c.n_heads;
  a.d_latent = c.d_latent;
  a.d_rope = c.d_rope;
  a.d_value = c.d_value;
  a.dense = 1;
  a.ring_rows = ring_rows(c);
  a.scale = 1.f / std::sqrt((float)(c.d_nope + c.d_rope));
  return cuda_status(launch_attn_simt(a, s));
}

vmla_status vmla_chunk_step_host(vmla_handle* h, int layer, const void* x_host, const void* q_host, void* out_host,
                                 const void* w_down, const void* w_uk, const void* w_uv, void* x_dev, void* q_dev,
                                 void* out_dev, int64_t first, int n, vmla_design design, void* stream) {
  vmla_status st = check_layer(h, layer);
  if (st != VMLA_OK) return st;
  if (!x_host || !q_host || !out_host || !x_dev || !q_dev || !out_dev) return VMLA_ERR_INVALID_ARG;
  if (n < 1 || n > h->cfg.chunk_frames) return VMLA_ERR_OUT_OF_RANGE;
  // everything the append and the attention would refuse is refused here, before any copy is enqueued
  int64_t new_F;
  if ((st = append_args(h, layer, x_dev, w_down, first, n, &new_F)) != VMLA_OK) return st;
  {
    vmla_design d = design;
    Window win;
    if ((st = attention_args(h, layer, q_dev, w_uk, w_uv, out_dev, first, n, &d, new_F, &win)) != VMLA_OK) return st;
  }
  if ((st = ensure_err(h)) != VMLA_OK) return st;
  const vmla_config& c = h->cfg;
  const size_t rows = (size_t)n * tokens_per_frame(c) * c.batch;
  const size_t xb = rows * c.d_model * esize(c);
  const size_t qb = rows * c.n_heads * (size_t)(c.d_nope + c.d_rope) * esize(c);
  const size_t ob = rows * c.n_heads * (size_t)c.d_value * sizeof(float);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (!h->copy_stream) {
    if ((e = cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&h->out_stream, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e);
    for (cudaEvent_t* ev : {&h->x_ready, &h->q_ready, &h->x_free, &h->q_free, &h->out_group, &h->out_done})
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return cuda_fail(e);
  }
  cudaStream_t cs = h->copy_stream;
  // inputs on the copy stream: x once the previous call's append has read x_dev, q once its
  // attention has read q_dev, so both copies overlap the previous call's attention and output
  // copy; the compute stream waits for each copy before its consumer
  if ((e = cudaStreamWaitEvent(cs, h->x_free, 0)) != cudaSuccess ||
      (e = cudaMemcpyAsync(x_dev, x_host, xb, cudaMemcpyHostToDevice, cs)) != cudaSuccess ||
      (e = cudaEventRecord(h->x_ready, cs)) != cudaSuccess || (e = cudaStreamWaitEvent(cs, h->q_free, 0)) != cudaSuccess ||
      (e = cudaMemcpyAsync(q_dev, q_host, qb, cudaMemcpyHostToDevice, cs)) != cudaSuccess ||
      (e = cudaEventRecord(h->q_ready, cs)) != cudaSuccess || (e = cudaStreamWaitEvent(s, h->x_ready, 0)) != cudaSuccess)
    return cuda_fail(e);
  if ((st = vmla_cache_append(h, layer, x_dev, w_down, first, n, stream)) != VMLA_OK) return st;
  if ((e = cudaEventRecord(h->x_free, s)) != cudaSuccess || (e = cudaStreamWaitEvent(s, h->q_ready, 0)) != cudaSuccess)
    return cuda_fail(e);
  // q_free is recorded as soon as the query-prep kernel has read q_dev, so the next call's q copy
  // overlaps this call's attention kernel
  HostOut hout{out_host, h->out_stream, h->out_group, h->out_done, false, h->q_free, false};
  if ((st = chunk_attention(h, layer, q_dev, w_uk, w_uv, out_dev, first, n, design, stream, &hout)) != VMLA_OK)
    return st;
  if (!hout.q_recorded && (e = cudaEventRecord(h->q_free, s)) != cudaSuccess) return cuda_fail(e);
  // the host result is there when `stream` is: the absorbed attention copied it back a group of
  // heads at a time (and made `stream` wait for the last copy); other paths copy it here
  if (hout.copied) return VMLA_OK;
  return cuda_status(cudaMemcpyAsync(out_host, out_dev, ob, cudaMemcpyDeviceToHost, s));
}

vmla_status vmla_device_status(vmla_handle* h, void* stream, uint32_t* flags) {
  if (!h) return VMLA_ERR_INVALID_ARG;
  unsigned* err = h->err ? h->err : device_error_word();
  if (!err) return VMLA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned v = 0;
  cudaError_t e;
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost)) != cudaSuccess) return cuda_fail(e);
  if (v && (e = cudaMemset(err, 0, sizeof(v))) != cudaSuccess) return cuda_fail(e);
  if (flags) *flags = v;
  if (v & DEV_ERR_BOUNDS_MASK) return VMLA_ERR_DEVICE_BOUNDS;
  if (v & DEV_ERR_RANGE) return VMLA_ERR_DEVICE_RANGE;
  if (v) return VMLA_ERR_DEVICE_TIMEOUT;
  return VMLA_OK;
}

vmla_status vmla_set_append_tiling(vmla_handle* h, int n_split, int row_tiles, int max_ctas) {
  if (!h || n_split < 0 || n_split > 2 || row_tiles < 0 || row_tiles > 2 || max_ctas < 0) return VMLA_ERR_INVALID_ARG;
  if (row_tiles == 2 && n_split == 2) return VMLA_ERR_INVALID_ARG;
  h->append_split = n_split;
  h->append_rows = row_tiles;
  h->append_ctas = max_ctas;
  return VMLA_OK;
}

const char* vmla_last_error_detail(void) { return g_detail; }

vmla_status vmla_profile_enable(vmla_handle* h, int enable) {
  if (!h) return VMLA_ERR_INVALID_ARG;
  h->profiling = enable != 0;
  for (auto& t : h->timers) t.used = 0;
  return VMLA_OK;
}

vmla_status vmla_profile_read(vmla_handle* h, int stage, double* total_ms, int* launches) {
  if (!h || stage < 0 || stage >= kStages || !total_ms || !launches) return VMLA_ERR_INVALID_ARG;
  auto& t = h->timers[stage];
  double sum = 0;
  for (size_t k = 0; k + 1 < t.used; k += 2) {
    if (cudaEventSynchronize(t.ev[k + 1]) != cudaSuccess) return VMLA_ERR_CUDA;
    float ms = 0;
    if (cudaEventElapsedTime(&ms, t.ev[k], t.ev[k + 1]) != cudaSuccess) return VMLA_ERR_CUDA;
    sum += ms;
  }
  *total_ms = sum;
  *launches = (int)(t.used / 2);
  return VMLA_OK;
}

vmla_status vmla_selftest_exp2(const float* x, float* y, int64_t n, void* stream) {
  if (!x || !y || n < 0 || (n & 1) || (reinterpret_cast<uintptr_t>(x) & 7) || (reinterpret_cast<uintptr_t>(y) & 7))
    return VMLA_ERR_INVALID_ARG;
  return cuda_status(launch_selftest_exp2(x, y, n, static_cast<cudaStream_t>(stream)));
}

vmla_status vmla_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns > 1000000000ull) return VMLA_ERR_INVALID_ARG;
  unsigned* err = device_error_word();
  if (!err) return VMLA_ERR_CUDA;
  return cuda_status(launch_selftest_wait(err, limit_ns, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
