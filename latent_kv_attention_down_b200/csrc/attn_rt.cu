// Reconstruct-in-tile chunk attention (sm_100a) [paperlayer Sec. 3, On-demand
// reconstruction; gist.it pt. 2]: the per-head keys and values are rebuilt
// from the latent cache inside every key tile,
//   K_h = [W_uk,h c | RoPE(k_R)],   V_h = W_uv,h c,
// and never leave the SM; the attention itself is the standard d_h = 128 one.
// It is the design the absorbed kernel is measured against: it does the
// reconstruction GEMM (2 * 128 * d_c * 224 flops per key tile and CTA) on top
// of the per-head attention.
//
// One CTA owns 128 query rows of one head of one sample; W_uk,h and W_uv,h stay
// in shared memory.  Per key tile j:
//   recon(j)  R^T = [W_uv,h; W_uk,h] c_j^T on the tensor core: TMEM lanes are
//             head dimensions, columns the tile's 128 keys (two M=128 GEMMs:
//             W_uv,h rows, and W_uk,h's 96 rows whose 32 missing rows read the
//             next buffer and land in lanes nobody reads)
//   convert   one warpgroup turns R^T into bf16 operand tiles: thread = head
//             dimension, its row of 128 keys is contiguous in both tiles --
//             K^T [96 dims x keys] (MN-major B of Q K^T) and V^T [128 dims x
//             keys] (K-major B of P V); the positional columns of K come from
//             the rotated k_R tile (TMA, K-major) as the last two k-steps
//   S = Q K^T, softmax, O += P V as in the absorbed kernel (two softmax
//   warpgroups, each half of the keys, lazy rescale).
// Tensor pipe order: recon(0) QK(0) recon(1) | PV(j) QK(j+1) recon(j+2) ...,
// so the softmax of tile j overlaps the reconstruction of tile j+1 and the
// V(j+1) conversion overlaps Q K^T(j+1).
//
//   warp 0     TMA: Q^, W_uk,h, W_uv,h once; latent chunks (2-slot ring of
//              [128 keys x 64]) and rotated k_R tiles (2 slots)
//   warp 1     tcgen05.mma issuer + TMEM owner
//   warps 4-7  converter: R^T -> K^T, V^T tiles
//   warps 8-15 softmax (two groups) and the epilogue
// TMEM: R_uv [0,128)  R_uk [128,256)  S [256,384)  O [384,512).
// Registers: 512 threads launch with 128 each; setmaxnreg gives 104 to the
// first warpgroup, 88 to the converter and 152 to each softmax warpgroup
// (63488 of 65536; per SM sub-partition 15872 of 16384).
#include "kernels.h"
#include "ptx.cuh"

namespace vmla {
namespace {

constexpr int kThreads = 512;
constexpr int BLK = 16384;  // [128 rows x 64 bf16] SW128 block

template <int DL>
struct RtCfg {
  static constexpr int CB = DL / 64;         // latent column blocks
  static constexpr int UK_BLK = 96 * 128;    // [96 rows x 64] block of W_uk,h
  static constexpr int O_WUK = 0;            // W_uk,h first: its last block's phantom rows read W_uv,h
  static constexpr int O_WUV = O_WUK + CB * UK_BLK;
  static constexpr int O_Q = O_WUV + CB * BLK;
  static constexpr int O_C = O_Q + 2 * BLK;  // 2 slots of [128 keys x 64 latent]
  static constexpr int O_KR = O_C + 2 * BLK;  // 2 slots of [128 keys x 32] SW64
  static constexpr int KR_BYTES = 128 * 64;
  static constexpr int KT_BLK = 96 * 128;     // K^T block: [96 dims x 64 keys]
  static constexpr int O_K = O_KR + 2 * KR_BYTES;
  static constexpr int O_V = O_K + 2 * KT_BLK;
  static constexpr int O_BARS = O_V + 2 * BLK;
  static constexpr int SMEM = O_BARS + 2560;
  static constexpr int O_PARK = O_C;  // fp32 output image (64 KB) over the chunk ring and K/V tiles
  static_assert(O_BARS - O_PARK >= 4 * BLK, "epilogue staging");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(O_WUV % 1024 == 0 && O_Q % 1024 == 0 && O_C % 1024 == 0 && O_KR % 1024 == 0 &&
                    O_K % 1024 == 0 && O_V % 1024 == 0,
                "operand alignment");
};

struct Bars {
  uint64_t q_full;
  uint64_t c_full[2], c_empty[2];
  uint64_t kr_full[2], kr_empty[2];
  uint64_t r_full, r_empty;
  uint64_t k_ready, k_free, v_ready;
  uint64_t s_full, p_full, pv_done;
  uint64_t o_final, drain;
  uint32_t tslot;
  int abort_flag;
  float red[2][2][128];
};
static_assert(sizeof(Bars) <= 2560, "barrier block");

constexpr uint32_t R_UV = 0, R_UK = 128, S_COL = 256, O_COL = 384;

__device__ __forceinline__ void setmaxnreg_dec104() { asm volatile("setmaxnreg.dec.sync.aligned.u32 104;"); }
__device__ __forceinline__ void setmaxnreg_dec88() { asm volatile("setmaxnreg.dec.sync.aligned.u32 88;"); }
__device__ __forceinline__ void setmaxnreg_inc152() { asm volatile("setmaxnreg.inc.sync.aligned.u32 152;"); }

__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// bf16 of 32 consecutive keys (k0 = 0, 32, 64, 96) into a row of a [rows x 128 keys] operand
// tile made of two [rows x 64 keys] SW128 blocks, blk_bytes apart
__device__ __forceinline__ void st_keys32(uint8_t* tile, int blk_bytes, int row, int k0, const uint32_t (&v)[32]) {
  uint8_t* base = tile + (k0 >> 6) * blk_bytes + row * 128;
  const int c0 = (k0 & 63) >> 3;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 w = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                               pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                               pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                               pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
    *reinterpret_cast<uint4*>(base + (((c0 + q) ^ (row & 7)) << 4)) = w;
  }
}

__device__ __forceinline__ void st_row32_f32(uint8_t* tile, int r, int c0, const uint32_t (&v)[32], float scale) {
  uint8_t* row = tile + (c0 >> 5) * BLK + r * 128;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<float4*>(row + ((j ^ (r & 7)) << 4)) =
        make_float4(__uint_as_float(v[4 * j]) * scale, __uint_as_float(v[4 * j + 1]) * scale,
                    __uint_as_float(v[4 * j + 2]) * scale, __uint_as_float(v[4 * j + 3]) * scale);
}

template <int DL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_rt_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_c,
                   const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_uk,
                   const __grid_constant__ CUtensorMap tm_uv, const __grid_constant__ CUtensorMap tm_out,
                   const AttnTc a) {
  using C = RtCfg<DL>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicOr(a.err, DEV_ERR_BOUNDS);
    return;
  }
  Bars* bars = reinterpret_cast<Bars*>(smem + C::O_BARS);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int m0 = mt * 128;
  const int n_tiles = (a.n_keys + 127) / 128;
  const Guard g{&bars->abort_flag, a.err, a.limit_ns};

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->c_full[s], 1);
      mbar_init(&bars->c_empty[s], 1);
      mbar_init(&bars->kr_full[s], 1);
      mbar_init(&bars->kr_empty[s], 1);
    }
    mbar_init(&bars->r_full, 1);
    mbar_init(&bars->r_empty, 4);
    mbar_init(&bars->k_ready, 4);
    mbar_init(&bars->k_free, 1);
    mbar_init(&bars->v_ready, 4);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_full, 8);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->o_final, 1);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tslot;

  if (warp < 4) {
    setmaxnreg_dec104();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      prefetch_tmap(&tm_c);
      prefetch_tmap(&tm_kr);
      mbar_arrive_expect_tx(&bars->q_full, 2 * BLK + C::CB * (C::UK_BLK + BLK));
      for (int blk = 0; blk < 2; ++blk)
        tma_load_3d(smem + C::O_Q + blk * BLK, &tm_q, &bars->q_full, blk * 64, m0, b * a.n_heads + h);
      for (int cb = 0; cb < C::CB; ++cb) {
        tma_load_3d(smem + C::O_WUK + cb * C::UK_BLK, &tm_uk, &bars->q_full, cb * 64, 0, h);
        tma_load_3d(smem + C::O_WUV + cb * BLK, &tm_uv, &bars->q_full, cb * 64, 0, h);
      }
      int cc = 0, kr_issued = 0;
      bool ok = true;
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int ks = j & 1;
        if (!(ok = wait_phase(&bars->kr_empty[ks], ((j >> 1) & 1) ^ 1, g, DEV_ERR_TIMEOUT_PRODUCER))) break;
        mbar_arrive_expect_tx(&bars->kr_full[ks], C::KR_BYTES);
        tma_load_3d(smem + C::O_KR + ks * C::KR_BYTES, &tm_kr, &bars->kr_full[ks], 0, j * 128, b);
        ++kr_issued;
        for (int cb = 0; cb < C::CB; ++cb, ++cc) {
          const int s = cc & 1;
          if (!(ok = wait_phase(&bars->c_empty[s], ((cc >> 1) & 1) ^ 1, g, DEV_ERR_TIMEOUT_PRODUCER))) break;
          mbar_arrive_expect_tx(&bars->c_full[s], BLK);
          tma_load_3d(smem + C::O_C + s * BLK, &tm_c, &bars->c_full[s], cb * 64, j * 128, b);
        }
      }
      if (bars->abort_flag) {
        drain_phase(&bars->q_full, 0, g);
        for (int i = cc > 2 ? cc - 2 : 0; i < cc; ++i) drain_phase(&bars->c_full[i & 1], (i >> 1) & 1, g);
        for (int i = kr_issued > 2 ? kr_issued - 2 : 0; i < kr_issued; ++i)
          drain_phase(&bars->kr_full[i & 1], (i >> 1) & 1, g);
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t s_base = smem_u32(smem);
      constexpr uint32_t id_r = idesc_bf16_f32(128, 128, false, false);   // A, B K-major
      constexpr uint32_t id_qk = idesc_bf16_f32(128, 128, false, true);   // B (K^T) MN-major
      constexpr uint32_t id_qr = idesc_bf16_f32(128, 128, false, false);  // B (rotated k_R) K-major
      const uint64_t q_d = smem_desc(s_base + C::O_Q, 16, 1024, LAYOUT_SW128);
      const uint64_t kt_d = smem_desc(s_base + C::O_K, C::KT_BLK, 1024, LAYOUT_SW128);
      const uint64_t vt_d = smem_desc(s_base + C::O_V, 16, 1024, LAYOUT_SW128);
      int cc = 0;
      // R^T = [W_uv; W_uk] c_j^T over the tile's latent chunks
      auto recon = [&](void) -> bool {
        for (int cb = 0; cb < C::CB; ++cb, ++cc) {
          const int s = cc & 1;
          if (!wait_phase(&bars->c_full[s], (cc >> 1) & 1, g, DEV_ERR_TIMEOUT_MMA)) return false;
          tc_fence_after();
          const uint64_t cd = smem_desc(s_base + C::O_C + s * BLK, 16, 1024, LAYOUT_SW128);
          const uint64_t uv = smem_desc(s_base + C::O_WUV + cb * BLK, 16, 1024, LAYOUT_SW128);
          const uint64_t uk = smem_desc(s_base + C::O_WUK + cb * C::UK_BLK, 16, 1024, LAYOUT_SW128);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            if (cb == 0 && kk == 0) {
              mma_ss_c<false>(tbase + R_UV, desc_add(uv, kk * 32), desc_add(cd, kk * 32), id_r);
              mma_ss_c<false>(tbase + R_UK, desc_add(uk, kk * 32), desc_add(cd, kk * 32), id_r);
            } else {
              mma_ss_c<true>(tbase + R_UV, desc_add(uv, kk * 32), desc_add(cd, kk * 32), id_r);
              mma_ss_c<true>(tbase + R_UK, desc_add(uk, kk * 32), desc_add(cd, kk * 32), id_r);
            }
          }
          mma_commit(&bars->c_empty[s]);
        }
        mma_commit(&bars->r_full);
        return true;
      };
      // S = Q^ K^T: 6 k-steps over the rebuilt content dims, 2 over the rotated positional dims
      auto qk = [&](int j) -> bool {
        if (!wait_phase(&bars->k_ready, j & 1, g, DEV_ERR_TIMEOUT_MMA) ||
            !wait_phase(&bars->kr_full[j & 1], (j >> 1) & 1, g, DEV_ERR_TIMEOUT_MMA))
          return false;
        tc_fence_after();
        const uint64_t kr_d = smem_desc(s_base + C::O_KR + (j & 1) * C::KR_BYTES, 16, 512, LAYOUT_SW64);
#pragma unroll
        for (int kk = 0; kk < 6; ++kk) {
          const uint64_t qa = desc_add(q_d, (kk >> 2) * BLK + (kk & 3) * 32);
          if (kk == 0)
            mma_ss_c<false>(tbase + S_COL, qa, desc_add(kt_d, kk * 2048), id_qk);
          else
            mma_ss_c<true>(tbase + S_COL, qa, desc_add(kt_d, kk * 2048), id_qk);
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_ss_c<true>(tbase + S_COL, desc_add(q_d, BLK + 64 + kk * 32), desc_add(kr_d, kk * 32), id_qr);
        mma_commit(&bars->s_full);
        mma_commit(&bars->kr_empty[j & 1]);
        mma_commit(&bars->k_free);
        return true;
      };
      bool ok = wait_phase(&bars->q_full, 0, g, DEV_ERR_TIMEOUT_MMA);
      ok = ok && recon() && qk(0);
      if (ok && n_tiles > 1) ok = wait_phase(&bars->r_empty, 0, g, DEV_ERR_TIMEOUT_MMA) && recon();
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (!(ok = wait_phase(&bars->p_full, j & 1, g, DEV_ERR_TIMEOUT_MMA) &&
                   wait_phase(&bars->v_ready, j & 1, g, DEV_ERR_TIMEOUT_MMA)))
          break;
        tc_fence_after();
        {
          constexpr uint32_t id_pv = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t vb = desc_add(vt_d, (kk >> 2) * BLK + (kk & 3) * 32);
            if (kk == 0 && j == 0)
              mma_ts_c<false>(tbase + O_COL, tbase + S_COL, vb, id_pv);
            else
              mma_ts_c<true>(tbase + O_COL, tbase + S_COL + kk * 8, vb, id_pv);
          }
        }
        mma_commit(&bars->pv_done);
        if (j + 1 < n_tiles && !(ok = qk(j + 1))) break;
        if (j + 2 < n_tiles && !(ok = wait_phase(&bars->r_empty, (j + 1) & 1, g, DEV_ERR_TIMEOUT_MMA) && recon()))
          break;
      }
      if (ok) mma_commit(&bars->o_final);
      if (bars->abort_flag) {
        mma_commit(&bars->drain);
        drain_phase(&bars->drain, 0, g);
      }
    }
  } else if (warp < 8) {
    setmaxnreg_dec88();
    // ------------------------------------------------------------ converter: R^T -> K^T, V^T
    const int wq = warp & 3;
    const int d = wq * 32 + lane;  // head dimension == TMEM lane
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(wq * 32) << 16);
    uint8_t* kt = smem + C::O_K;
    uint8_t* vt = smem + C::O_V;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      ok = ok && __all_sync(0xffffffffu, wait_phase(&bars->r_full, j & 1, g, DEV_ERR_TIMEOUT_SOFTMAX));
      if (j > 0) ok = ok && __all_sync(0xffffffffu, wait_phase(&bars->k_free, (j - 1) & 1, g, DEV_ERR_TIMEOUT_SOFTMAX));
      if (ok && wq < 3) {  // content dims 0..95 of K; lanes 96..127 of R_uk hold nothing
        tc_fence_after();
#pragma unroll 1
        for (int k0 = 0; k0 < 128; k0 += 32) {
          uint32_t v[32];
          tmem_ld32(lane_base + R_UK + k0, v);
          st_keys32(kt, C::KT_BLK, d, k0, v);
        }
      }
      fence_async_smem();
      tc_fence_before();
      warp_arrive(&bars->k_ready);
      if (j > 0) ok = ok && __all_sync(0xffffffffu, wait_phase(&bars->pv_done, (j - 1) & 1, g, DEV_ERR_TIMEOUT_SOFTMAX));
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int k0 = 0; k0 < 128; k0 += 32) {
          uint32_t v[32];
          tmem_ld32(lane_base + R_UV + k0, v);
          st_keys32(vt, BLK, d, k0, v);
        }
      }
      fence_async_smem();
      tc_fence_before();
      warp_arrive(&bars->v_ready);
      warp_arrive(&bars->r_empty);
    }
  } else {
    setmaxnreg_inc152();
    // ------------------------------------------------------------ softmax and epilogue
    const int wg = (warp - 8) >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(wq * 32) << 16);
    constexpr int HS = 64;
    const int sc0 = wg * HS;
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      ok = ok && __all_sync(0xffffffffu, wait_phase(&bars->s_full, j & 1, g, DEV_ERR_TIMEOUT_SOFTMAX));
      uint32_t sraw[HS];
      float mx = -INFINITY;
      if (ok) {
        tc_fence_after();
        tmem_ld64(lane_base + S_COL + sc0, sraw);
        const int valid = a.n_keys - j * 128 - sc0;
        if (valid < HS) {
#pragma unroll
          for (int c = 0; c < HS; ++c)
            if (c >= valid) sraw[c] = __float_as_uint(-INFINITY);
        }
        float mxc[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t* v = &sraw[16 * k];
          float m = max3f(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
          for (int i = 3; i < 15; i += 2) m = max3f(m, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
          mxc[k] = fmaxf(m, __uint_as_float(v[15]));
        }
        mx = fmaxf(fmaxf(mxc[0], mxc[1]), fmaxf(mxc[2], mxc[3]));
      }
      bars->red[j & 1][wg][r] = mx;
      named_bar_sync(2, 256);
      const float m_tile = fmaxf(mx, bars->red[j & 1][wg ^ 1][r]) * a.scale_log2;
      if (ok) {
        if (j == 0) {
          m_run = m_tile;
        } else if (__any_sync(0xffffffffu, m_tile > m_run + a.rescale_threshold)) {
          const float m_new = fmaxf(m_run, m_tile);
          const float alpha = ex2_approx(m_run - m_new);
          ok = __all_sync(0xffffffffu, wait_phase(&bars->pv_done, (j - 1) & 1, g, DEV_ERR_TIMEOUT_SOFTMAX));
          if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int c = wg * 64; c < wg * 64 + 64; c += 32) {
              uint32_t o[32];
              tmem_ld32(lane_base + O_COL + c, o);
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st32(lane_base + O_COL + c, o);
            }
            l_run *= alpha;
            m_run = m_new;
          }
        }
      }
      if (ok) {
        const float2 nm2 = make_float2(-m_run, -m_run);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        uint32_t packed[HS / 2];
#pragma unroll
        for (int k = 0; k < HS / 2; ++k) {
          const float2 y =
              __ffma2_rn(make_float2(__uint_as_float(sraw[2 * k]), __uint_as_float(sraw[2 * k + 1])), sc2, nm2);
          const float2 pr = exp2_mixed(y, k);
          acc[k & 3] = __fadd2_rn(acc[k & 3], pr);
          packed[k] = pack_bf16x2(pr.x, pr.y);
        }
        tmem_st32(lane_base + S_COL + wg * (HS / 2), packed);
        const float2 acc4 = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
        l_run += acc4.x + acc4.y;
        tc_fence_before();
      }
      warp_arrive(&bars->p_full);
    }
    ok = ok && __all_sync(0xffffffffu, wait_phase(&bars->o_final, 0, g, DEV_ERR_TIMEOUT_EPILOGUE));
    bars->red[n_tiles & 1][wg][r] = l_run;
    named_bar_sync(2, 256);
    const float inv_l = 1.f / (l_run + bars->red[n_tiles & 1][wg ^ 1][r]);
    // every MMA has completed and the converter is done: park the fp32 rows over the ring and tiles
    uint8_t* park = smem + C::O_PARK;
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int c = wg * 64; c < wg * 64 + 64; c += 32) {
        uint32_t o[32];
        tmem_ld32(lane_base + O_COL + c, o);
        st_row32_f32(park, r, c, o, inv_l);
      }
    }
    fence_async_smem();
    named_bar_sync(1, 256);
    if (wg == 0 && r == 0 && ok && !bars->abort_flag) {
      for (int blk = 0; blk < 4; ++blk) tma_store_3d(&tm_out, park + blk * BLK, h * 128 + blk * 32, m0, b);
      bulk_commit();
      bulk_wait_all_read();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <int DL>
cudaError_t go_rt(const CUtensorMap& tq, const CUtensorMap& tc, const CUtensorMap& tkr, const CUtensorMap& tuk,
                  const CUtensorMap& tuv, const CUtensorMap& to, const AttnTc& a, int batch, cudaStream_t s) {
  using C = RtCfg<DL>;
  static const cudaError_t attr =
      cudaFuncSetAttribute(attn_rt_kernel<DL>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (attr != cudaSuccess) return attr;
  if (a.n_q <= 0 || a.n_keys <= 0) return cudaSuccess;
  attn_rt_kernel<DL><<<dim3(a.m_tiles, a.n_heads, batch), kThreads, C::SMEM, s>>>(tq, tc, tkr, tuk, tuv, to, a);
  return cudaGetLastError();
}

}  // namespace

bool attn_reconstruct_supported(int d_latent) { return d_latent == 64 || d_latent == 128 || d_latent == 192; }

cudaError_t launch_attn_reconstruct_tc(int d_latent, const CUtensorMap& tq, const CUtensorMap& tc,
                                       const CUtensorMap& tkr, const CUtensorMap& tuk, const CUtensorMap& tuv,
                                       const CUtensorMap& to, const AttnTc& a, int batch, cudaStream_t s) {
  switch (d_latent) {
    case 64: return go_rt<64>(tq, tc, tkr, tuk, tuv, to, a, batch, s);
    case 128: return go_rt<128>(tq, tc, tkr, tuk, tuv, to, a, batch, s);
    case 192: return go_rt<192>(tq, tc, tkr, tuk, tuv, to, a, batch, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace vmla
