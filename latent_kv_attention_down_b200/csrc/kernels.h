// Internal interface between the host library (vmla.cpp) and the CUDA kernels.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "vmla.h"

namespace vmla {

constexpr int kMaxPairs = 64;  // rotary pairs (d_rope up to 128)

// Bits of the library's device status word.
enum DeviceError : unsigned {
  DEV_ERR_TIMEOUT_PRODUCER = 1u << 0,
  DEV_ERR_TIMEOUT_MMA = 1u << 1,
  DEV_ERR_TIMEOUT_SOFTMAX = 1u << 2,
  DEV_ERR_TIMEOUT_EPILOGUE = 1u << 3,
  DEV_ERR_TIMEOUT_SELFTEST = 1u << 4,
  DEV_ERR_BOUNDS = 1u << 5,
  DEV_ERR_RANGE = 1u << 6,  // a value past the range of its storage type (fp16 per-head operands)
};
constexpr unsigned DEV_ERR_BOUNDS_MASK = DEV_ERR_BOUNDS;

// 3D-RoPE: pair p < n_t turns with the frame index t, then n_h pairs with the
// grid row h, then n_w pairs with the grid column w, by position * freq[p].
struct Rope {
  float freq[kMaxPairs];
  int n_t, n_h, n_w;
};

// Ring geometry of one sample's cache: frame f lives in ring frame slot f mod W.
struct Ring {
  int tokens_per_frame;  // T_f
  int grid_w;
  int window_frames;     // W, sink included
  int sink_frames;       // S: frames 0..S-1 keep slots 0..S-1; later frames rotate through S..W-1
};

// Ring slot of frame f: a sink frame keeps its own slot, any other frame takes the slot
// of the local frame it evicts (the oldest) [paperlayer App. D.4].
__host__ __device__ inline int64_t ring_frame_slot(const Ring& g, int64_t f) {
  return f < g.sink_frames ? f : g.sink_frames + (f - g.sink_frames) % (g.window_frames - g.sink_frames);
}
// Window-relative t of the keys in ring slot `slot` [paperlayer App. D.5]: sink slots keep
// t = slot; local slots count from the oldest local frame, whose slot is S + local_start_slot.
__host__ __device__ inline int ring_slot_t(const Ring& g, int slot, int local_start_slot) {
  if (slot < g.sink_frames) return slot;
  const int L = g.window_frames - g.sink_frames;
  return g.sink_frames + (slot - g.sink_frames - local_start_slot + L) % L;
}

// ------------------------------------------------------------------ fp32 SIMT path (any shape)
struct SimtAppend {
  const float* x;       // [B][rows][D]
  const float* w_down;  // [d_c + d_r][D]
  float* ckv;           // [B][W*T_f][d_c]   (or a contiguous [B][rows][d_c] scratch)
  float* kr;            // [B][W*T_f][d_r]
  int batch, rows, d_model, d_latent, d_rope;
  int64_t first_frame;
  int rotate;           // rotate k_R with the absolute frame index before storing
  int contiguous;       // store row m at row m (scratch) instead of its ring slot
  int64_t out_rows;     // rows per sample of ckv/kr
  Ring ring;
  Rope rope;
};
cudaError_t launch_append_simt(const SimtAppend& a, cudaStream_t s);

struct RopeWindow {  // rotate the window's positional keys with window-relative t
  const void* kr;    // [B][W*T_f][d_r]  (bf16 path: bf16)
  void* kr_rot;      // [B][W*T_f][d_r]  (bf16 path: bf16)
  int batch, n_keys, d_rope;
  int window_start_slot;  // (ring slot of the oldest local frame) - sink_frames
  Ring ring;
  Rope rope;
};
cudaError_t launch_rope_window_f32(const RopeWindow& a, cudaStream_t s);
cudaError_t launch_rope_window_bf16(const RopeWindow& a, cudaStream_t s);

struct SimtQPrep {  // q~ = [W_uk^T q_nope | RoPE(q_rope)]  (absorbed) or [q_nope | RoPE(q_rope)] (dense)
  const float* q;     // [B][n_q][n_h][d_nope + d_r]
  const float* w_uk;  // [n_h][d_nope][d_c]   (unused when absorb == 0)
  float* qt;          // [B][n_h][n_q][width]
  int batch, n_q, n_heads, d_nope, d_rope, d_latent, absorb;
  int64_t t_first;    // frame index t of query row 0
  Ring ring;
  Rope rope;
};
cudaError_t launch_qprep_simt(const SimtQPrep& a, cudaStream_t s);

struct SimtAttn {
  const float* qt;    // [B][n_h][n_q][dqk]
  const float* key;   // latent: [B][ring_rows][d_c] (+ kpos [B][ring_rows][d_r]); dense: [B][ring_rows][2][n_h][dv]
  const float* kpos;  // rotated positional keys (latent only)
  const float* w_uv;  // [n_h][dv][d_c] (latent only)
  float* out;         // [B][n_q][n_h*dv]
  int batch, n_q, n_keys, n_heads, d_latent, d_rope, d_value, dense;
  int64_t ring_rows;
  float scale;        // 1/sqrt(d_nope + d_rope)
};
cudaError_t launch_attn_simt(const SimtAttn& a, cudaStream_t s);

struct SimtDenseReconstruct {  // dense per-head entries from a chunk's latents
  const float* c;       // [B][rows][d_c]  (contiguous scratch)
  const float* r;       // [B][rows][d_r]  (unrotated)
  const float* w_uk;    // [n_h][d_nope][d_c]
  const float* w_uv;    // [n_h][dv][d_c]
  float* dense;         // [B][W*T_f][2][n_h][dv]
  int batch, rows, n_heads, d_nope, d_rope, d_latent, d_value;
  int64_t first_frame;
  Ring ring;
  Rope rope;
};
cudaError_t launch_dense_reconstruct_simt(const SimtDenseReconstruct& a, cudaStream_t s);

// ------------------------------------------------------------------ bf16 tcgen05 path (sm_100a)
struct AppendTc {
  __nv_bfloat16* ckv;  // [B][ring_rows][d_c] or contiguous [B][rows][d_c + d_r] when contiguous
  __nv_bfloat16* kr;   // [B][ring_rows][d_r]
  int rows, d_model, d_latent, d_rope;  // d_rope 16, 32 or 64
  int64_t first_frame;
  int rotate, contiguous;
  int64_t ring_rows;
  Ring ring;
  Rope rope;
  unsigned* err;
  uint64_t limit_ns;
};
// Work split of the persistent append kernel for a call: `parts` column parts
// of [c_KV | k_R] (1, 2 or 3), `row_tiles` 128-row tiles per work item (1 or 2;
// 2 only with one part) and a grid cap `ctas` (0: one CTA per SM).  n_split 0
// chooses two parts when the 128-row tiles alone would leave SMs idle (and
// always past 256 columns); past 512 columns there are always three.  row_tiles
// 0 takes one row tile (two measured slower).
// Columns of one part when [c_KV | k_R] (n_out columns) is split in `parts`: a multiple of 16
// (the MMA's N); the last part may run past n_out (those rows of W_down read as zeros).
constexpr int append_part_cols(int n_out, int parts) { return (n_out + 16 * parts - 1) / (16 * parts) * 16; }

struct AppendPlan {
  int parts, ctas, row_tiles;
};
AppendPlan append_tc_plan(int n_out, int rows, int batch, int n_split, int row_tiles, int ctas);
// x map: 3D (D, rows, B) box (64,128,1) SW128; w map: 2D (D, n_out) box (64, append_part_cols(n_out, parts))
// SW128, n_out = d_c + d_rope.
cudaError_t launch_append_tc(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const AppendTc& a, int batch,
                             cudaStream_t s, const AppendPlan& plan);

struct QPrepTc {
  const __nv_bfloat16* q;  // [B][n_q][n_h][128]: per head d_nope = 128 - d_rope content dims, then d_rope
  __nv_bfloat16* qt;       // [B][n_h][n_q][d_c + d_rope]
  int n_q, n_heads, d_latent, d_rope;  // d_rope 16, 32 or 64
  int64_t t_first;
  Ring ring;
  Rope rope;
  unsigned* err;
  uint64_t limit_ns;
};
// q map: 3D (n_h*128, n_q, B) box (64,128,1) SW128; w_uk map: 3D (d_c, d_nope, n_h) box (64, d_nope, 1)
// SW128; out map (the stores of qt): 3D (d_c + d_rope, n_q, B*n_h) box (64, 64, 1) SW128
cudaError_t launch_qprep_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_wuk, const CUtensorMap& tm_out,
                            const QPrepTc& a, int batch, cudaStream_t s);

// Query-latent absorption: qt [B][n_h][n_q][d_c + d_rope] = [A_h ; W_qr,h] c_Q, positional part
// rotated at the query positions.  c_Q map: 3D (d_q, n_q, B) box (64,128,1) SW128; weight map:
// 3D (d_q, d_c + d_rope, n_h) box (64, d_c + d_rope, 1) SW128; out map as for launch_qprep_tc.
// d_latent 64, 128 or 192, d_rope 16, 32, 64 or 96 with d_latent + d_rope <= 256; d_q % 64 == 0.
struct QLatTc {
  __nv_bfloat16* qt;
  int n_q, n_heads, d_latent, d_rope, d_q;
  int64_t t_first;
  Ring ring;
  Rope rope;
  unsigned* err;
  uint64_t limit_ns;
};
bool qlat_supported(int d_latent, int d_rope, int d_q);
cudaError_t launch_qlat_tc(const CUtensorMap& tm_cq, const CUtensorMap& tm_w, const CUtensorMap& tm_out,
                           const QLatTc& a, int batch, cudaStream_t s);
// w_qabs [n_h][d_c + d_rope][d_q] = [W_uk,h^T W_uq,h ; W_qr,h]
cudaError_t launch_fold_query(const __nv_bfloat16* w_uq, const __nv_bfloat16* w_qr, const __nv_bfloat16* w_uk,
                              __nv_bfloat16* w_qabs, int n_heads, int d_nope, int d_rope, int d_c, int d_q,
                              cudaStream_t s);

struct AttnTc {
  int n_q, n_keys, n_heads, m_tiles;
  float scale_log2;  // log2(e) / sqrt(d_nope + d_rope)
  float rescale_threshold;  // lazy-rescale threshold of the running max, log2 units
  unsigned* err;
  uint64_t limit_ns;
  int h0 = 0;       // absorbed and dense attention: first head of this launch
  int h_count = 0;  // heads of this launch (grid y); 0 = all n_heads
};
// Absorbed design.  qt maps: 3D (d_c+32, n_q, B*n_h): latent box (64,128,1) SW128, rope box (32,128,1) SW64;
// ckv map: 3D (d_c, n_keys, B) box (64,BN,1) SW128; kr map: 3D (32, n_keys, B) box (32,BN,1) SW64;
// w_uv map: 3D (d_c, 128, n_h) box (64,128,1) SW128; out map: 3D (n_h*128, n_q, B) box (64,128,1) SW128.
// d_rope 16, 32, 64 or 96 (64 and 96 up to d_latent 192): tm_qr / tm_kr boxes are d_rope wide, swizzled
// at d_rope * 2 bytes (32B, 64B or 128B), except for 96: boxes 32 wide, SW64 (three loads per tile)
bool attn_absorbed_supported(int d_latent, int d_rope);
cudaError_t launch_attn_absorbed_tc(int d_latent, int d_rope, const CUtensorMap& tm_q, const CUtensorMap& tm_qr,
                                    const CUtensorMap& tm_ckv, const CUtensorMap& tm_kr, const CUtensorMap& tm_wuv,
                                    const CUtensorMap& tm_out, const AttnTc& a, int batch, cudaStream_t s);
int attn_absorbed_block_n(int d_latent);  // keys per tile (TMA box rows of the key maps)

// Absorbed attention that stores O_bar = softmax-weighted latents / l (per head, d_c wide) as a
// bf16 pair instead of applying W_uv,h: maps 3D (n_h*d_c, n_q, B) bf16 box (64,128,1) SW128 for
// the rounded part (tob_hi) and the residual (tob_lo).
cudaError_t launch_attn_absorbed_obar_tc(int d_latent, int d_rope, const CUtensorMap& tm_q, const CUtensorMap& tm_qr,
                                         const CUtensorMap& tm_ckv, const CUtensorMap& tm_kr,
                                         const CUtensorMap& tob_hi, const CUtensorMap& tob_lo, const AttnTc& a,
                                         int batch, cudaStream_t s);

// Folded output mixer: out [rows][n_out] fp32 = (O_bar hi + lo) [rows][k] x w_fold[n_out][k]^T.
// Maps 3D with a unit last extent: hi/lo (k, rows, 1) bf16 box (64,128,1) SW128; w_fold (k, n_out, 1)
// box (64,128,1) SW128; out (n_out, rows, 1) fp32 box (32,128,1) SW128.  k % 64 == 0, n_out % 128 == 0.
struct FoldTc {
  int rows, k, n_out;
  unsigned* err;
  uint64_t limit_ns;
};
cudaError_t launch_fold_gemm_tc(const CUtensorMap& tm_hi, const CUtensorMap& tm_lo, const CUtensorMap& tm_w,
                                const CUtensorMap& tm_out, const FoldTc& a, cudaStream_t s);
// w_fold [d_out][n_h*d_c] = W_O,h W_uv,h side by side (w_o [d_out][n_h*d_v], w_uv [n_h][d_v][d_c]).
cudaError_t launch_fold_weights(const __nv_bfloat16* w_o, const __nv_bfloat16* w_uv, __nv_bfloat16* w_fold, int d_out,
                                int n_heads, int d_v, int d_c, cudaStream_t s);

// Reconstruct-in-tile design (attn_rt.cu), d_latent 64, 128 or 192.  q map: dense queries
// 3D (128, n_q, B*n_h) box (64,128,1) SW128; ckv map box (64,128,1) SW128; kr map box (32,128,1)
// SW64; w_uk map 3D (d_c, 96, n_h) box (64,96,1); w_uv map box (64,128,1); out fp32 box (32,128,1).
bool attn_reconstruct_supported(int d_latent);
cudaError_t launch_attn_reconstruct_tc(int d_latent, const CUtensorMap& tm_q, const CUtensorMap& tm_ckv,
                                       const CUtensorMap& tm_kr, const CUtensorMap& tm_wuk, const CUtensorMap& tm_wuv,
                                       const CUtensorMap& tm_out, const AttnTc& a, int batch, cudaStream_t s);
int attn_dense_block_n();

// Dense per-head attention, d_head = 128.  q map: 3D (128, n_q, B*n_h) box (64,128,1);
// kv map: 3D (2*n_h*128, n_keys, B) box (64,128,1); out: 3D fp32 (n_h*128, n_q, B) box (32,128,1) SW128.
// f16: q and kv hold fp16 (the reconstruct-once workspace) instead of bf16 (the dense cache).
cudaError_t launch_attn_dense_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const CUtensorMap& tm_out,
                                 const AttnTc& a, int batch, cudaStream_t s, bool f16);

struct DenseQTc {  // q' = [q_nope | RoPE(q_rope)] -> [B][n_h][n_q][128]
  const __nv_bfloat16* q;
  void* qd;                         // bf16, or fp16 when f16
  int batch, n_q, n_heads, d_rope;  // d_rope a multiple of 8: the last d_rope of a head's 128 dims
  int64_t t_first;
  Ring ring;
  Rope rope;
  int f16 = 0;            // write fp16 (DEV_ERR_RANGE in *err for a value past 65504)
  unsigned* err = nullptr;
};
cudaError_t launch_dense_q_bf16(const DenseQTc& a, cudaStream_t s);

struct ReconTc {  // per-head dense entries from latents (tcgen05)
  const void* kr;           // positional keys [B][kr_rows][d_rope], bf16; unrotated when rotate or
                            // window_t is set
  void* dense;              // [B][ring_rows][2][n_h][128], bf16 or (f16) fp16
  int f16;                  // fp16 entries (DEV_ERR_RANGE for a value past 65504)
  int rows, n_heads, d_latent, d_rope;  // d_rope 16, 32, 64 or 96 (d_nope = 128 - d_rope)
  int64_t first_frame;      // frame of row 0 (ring placement and absolute t)
  int rotate;               // rotate kr with the absolute frame index
  int to_ring;              // 1: row m -> ring slot of its frame; 0: row m -> row m
  int window_t = 0;         // rotate kr with the window-relative t of row m's ring slot (to_ring 0)
  int window_start_slot = 0;  // (ring slot of the oldest local frame) - sink_frames, for window_t
  int64_t kr_rows;          // rows per sample of kr
  int kr_stride;            // elements between consecutive kr rows
  int64_t ring_rows;        // rows per sample of dense
  Ring ring;
  Rope rope;
  unsigned* err;
  uint64_t limit_ns;
};
// c map: 3D (d_c, rows, B) box (64,128,1) SW128; w_uk map: 3D (d_c, d_nope, n_h) box (64,d_nope,1);
// w_uv map: 3D (d_c, 128, n_h) box (64,128,1).  f16 (the reconstruct-once window, to_ring 0) also
// needs tm_out: 3D fp16 (2*n_h*128, rows, B) over `dense`, box (64,128,1) SW128 (its row extent
// clips the last tile); the bf16 dense cache passes NULL.
cudaError_t launch_recon_tc(const CUtensorMap& tm_c, const CUtensorMap& tm_wuk, const CUtensorMap& tm_wuv,
                            const CUtensorMap* tm_out, const ReconTc& a, int batch, cudaStream_t s);

// ------------------------------------------------------------------ device status
unsigned* device_error_word();  // address of the library's device status word (current device)
cudaError_t launch_selftest_wait(unsigned* err, uint64_t limit_ns, cudaStream_t s);
// y[i] = the attention kernels' polynomial 2^x[i] (exp2_poly2), n even, 8-byte aligned arrays.
cudaError_t launch_selftest_exp2(const float* x, float* y, int64_t n, cudaStream_t s);

// ------------------------------------------------------------------ host helpers (vmla.cpp), shared by
// the entry points of every host file
Rope make_rope(const vmla_config& c);  // pair frequencies theta^(-2i/B_a), t pairs first
Ring make_ring(const vmla_config& c);

// The active context after F frames [paperlayer App. D.4, D.5]: ring slots [0, n_keys / T_f);
// a local frame f has window-relative t = f - t_origin, a sink frame t = f.
struct Window {
  int64_t t_origin;
  int64_t local_start;  // oldest local frame
  int n_keys;
  int start_slot;       // ring slot of the oldest local frame, minus sink_frames
};
Window window_of(const vmla_config& c, int64_t F);

// 3D TMA tensor map: dims (d0 innermost, d1, d2), byte strides s1, s2, box (b0, b1, 1); false when the
// driver refuses it (or its encoder entry point is missing).
bool map3(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
          uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw, CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
bool map2(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t s1, uint32_t b0, uint32_t b1,
          CUtensorMapSwizzle sw);

}  // namespace vmla
