// Chunk attention on tcgen05 tensor cores (sm_100a).
//
// Absorbed design [paperlayer App. E]: with W_uk folded into the query
// (q~_h = [W_uk,h^T q_nope,h | RoPE(q_rope,h)]), every head scores the SAME
// shared key [c_KV | RoPE(k_R)] (d_latent + d_rope wide) and accumulates the SAME
// shared values c_KV (d_latent wide): multi-query attention over the latent
// cache.  W_uv,h is applied once per output row after the softmax-weighted
// sum (value-path absorption), fused into the epilogue as a second tcgen05
// GEMM whose A operand is O_bar split into a bf16 pair (rounded + residual),
// so the only roundings left on the output path are the cache's, P's and
// q~'s.  The output is written in fp32.  The dense variant runs the same
// pipeline with per-head 128-wide K and V tiles (the 3072-scalar layout).
//
// One CTA owns 128 query rows of one head of one sample and streams the whole
// window in tiles of BN keys:
//   warp 0      TMA producer: the query tile once, then K/V tiles into a ring
//   warp 1      TMEM owner; tcgen05.mma issuer (one thread) of the absorbed design
//   warps 2, 3  per-head tiles: the Q K^T and the P V issuers (one thread each)
//   warps 4-11  two softmax warpgroups; thread r of either group owns query
//               row r = TMEM lane r, each group half of every tile's keys
// TMEM (512 columns): S0 [0,BN), S1 [BN,2BN), O [2BN, 2BN+DV).
//   S_j = Q K_j^T (fp32) lands in S[j&1]; the softmax threads turn it into
//   P_j = exp2(S_j * scale*log2e - m) as bf16 pairs written back over S[j&1];
//   O += P_j V_j reads P straight from TMEM (A operand) and V from the same
//   shared-memory tile as K (MN-major descriptor), so V is never loaded twice.
//   While the softmax works on S_j, the tensor core computes S_{j+1}; S_{j+2}
//   reuses S[j&1] once P V_j has read P_j (in-order tensor pipe).  Letting QK
//   run further ahead would need a third resident K/V tile, and the 227 KB of
//   shared memory then leave no room to prefetch the next one.
// Per-head tiles (d_head 128) take 192 keys per tile (S0, S1 of 192 columns,
//   O at 384) and release the K and V halves of a stage separately.
// The running max is only raised when it grows by more than 2^threshold (lazy
// rescale, 2^8 by default); O is then rescaled in TMEM after the previous P V
// has finished.  Every mbarrier wait is bounded; a CTA that gives up records
// the error and drains its in-flight copies and MMAs before releasing TMEM.
#include "kernels.h"
#include "ptx.cuh"

namespace vmla {
namespace {

constexpr int kThreads = 384;  // warp 0 TMA, warp 1 MMA + TMEM, warps 4-11 two softmax warpgroups
constexpr int kMaxStages = 6;
constexpr int kSoftmaxWarps = 8;

struct Bars {
  uint64_t q_full;
  uint64_t kv_full[kMaxStages];   // the stage's tile landed (per-head tiles: its K half)
  uint64_t kv_empty[kMaxStages];  // the stage may be reloaded (per-head tiles: its K half)
  uint64_t v_full[kMaxStages];    // per-head tiles: the stage's V half landed
  uint64_t v_empty[kMaxStages];   // per-head tiles: the stage's V half may be reloaded
  uint64_t s_full[3];  // S_j computed (MMA commit), by S buffer j % NSB
  uint64_t p_full[3];  // P_j stored over S_j by every softmax warp
  uint64_t p_done[3];  // P V_j has completed (MMA commit)
  uint64_t o_final;
  uint64_t wuv_full;
  uint64_t ob_full;
  uint64_t epi_done;
  uint64_t drain;
  uint64_t drain_pv;  // per-head tiles: the P V issuer's own drain
  uint32_t tslot;
  int abort_flag;
  float red[2][2][128];  // per-tile half-row maxima of the two softmax groups (tile parity, group, row)
};

template <int DL_, bool DENSE_, int DR_ = 32, bool F16_ = false>
struct AttnCfg {
  static constexpr bool DENSE = DENSE_;
  // per-head operands (Q, K, V and P) in fp16 instead of bf16: the reconstruct-once workspace
  static constexpr bool F16 = F16_;
  static_assert(!F16 || DENSE, "fp16 operands: per-head tiles only");
  static constexpr int DL = DL_;
  static constexpr int DR = DR_;                     // rotary dims of the shared key (absorbed)
  static constexpr int DQK = DENSE ? 128 : DL + DR;  // contraction width of S = Q K^T
  static constexpr int DV = DENSE ? 128 : DL;
  // keys per tile: 192 for per-head tiles (the softmax's fixed cost per tile -- loading S, the
  // row max and its exchange, handing P over -- is spread over 1.5x the keys; TMEM holds two
  // 192-column S buffers and O), 128 for the absorbed design's wider O
  static constexpr int BN = DENSE ? 192 : 128;
  static constexpr int QB = DENSE ? 2 : DL / 64;  // 64-wide SW128 blocks of a query or key row
  // the rotary columns sit in NRB blocks of RB bytes per row, each swizzled at its width: one block
  // of DR * 2 bytes for 16, 32 or 64 rotary dims, three 64-byte blocks for 96
  static constexpr int NRB = DENSE ? 0 : (DR == 96 ? 3 : 1);
  static constexpr int RB = DENSE ? 0 : (DR == 96 ? 64 : DR * 2);
  static constexpr uint32_t R_LAYOUT = RB == 128 ? LAYOUT_SW128 : (RB == 64 ? LAYOUT_SW64 : LAYOUT_SW32);
  static constexpr int Q_BYTES = QB * 16384 + NRB * 128 * RB;
  static constexpr int KBLK = BN * 128;           // one [BN keys x 64] SW128 block
  static constexpr int STAGE_BYTES = DENSE ? 4 * KBLK : QB * KBLK + NRB * BN * RB;
  static constexpr int SMEM_CAP = 232448;
  static constexpr int BARS = (sizeof(Bars) + 127) / 128 * 128;
  static constexpr int STAGES_FIT = (SMEM_CAP - BARS - Q_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > kMaxStages ? kMaxStages : STAGES_FIT;
  // S buffers: S_j (and P_j over it) in buffer j % NSB at S_COL + (j % NSB) * BN: two, Q K^T one
  // tile ahead of the softmax.  Per-head tiles have their K and V halves on barriers of their own
  // (K_j is free once Q K_j^T is done, V_j once P V_j is), so a K tile is never held back by the
  // P V of an older one.
  static constexpr int NSB = 2;
  static constexpr int S_COL = 0;
  static constexpr int O_COL = NSB * BN;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int SMEM = Q_BYTES + STAGES * STAGE_BYTES + BARS;
  // epilogue images: O_bar rounded over the query tile; W_uv,h in the ring stage that tile n_tiles
  // would have used (free two tiles before the end, so its load hides behind the last tiles), the
  // O_bar residual in the stage after it
  static_assert(STAGES >= 2, "the K/V ring needs two stages");
  static_assert(O_COL + DV <= 512, "TMEM budget");
  static_assert(SMEM <= SMEM_CAP, "shared memory budget");
  static_assert((DENSE || STAGE_BYTES >= DV * 256) && STAGES * STAGE_BYTES >= 65536, "epilogue staging");
  static_assert(DV % 64 == 0 && DV <= 256 && BN % 32 == 0, "tile shapes");
  static_assert(DENSE || DR == 16 || DR == 32 || DR == 64 || DR == 96, "rotary blocks of 32, 64 or 128 bytes per row");
};

// bf16 row of 32 floats into a 128B-swizzled K-major tile: row r, columns c0..c0+31
// (c0 a multiple of 32) of a tile made of [128 rows x 64 cols] blocks of 16 KB.
// With `lo` set, what is stored is the rounding residual v*scale - bf16(v*scale),
// so that hi + lo carries the value to about 16 significant bits.
__device__ __forceinline__ void st_swizzled_row32(uint8_t* tile, int r, int c0, const float (&v)[32], float scale,
                                                  bool lo) {
  uint8_t* blk = tile + (c0 >> 6) * 16384 + r * 128;
  const int j0 = (c0 & 63) >> 3;  // first 16-byte chunk of the 64-col block
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = v[8 * q + 2 * k] * scale, b = v[8 * q + 2 * k + 1] * scale;
      const uint32_t hi = pack_bf16x2(a, b);
      w[k] = lo ? pack_bf16x2(a - __uint_as_float(hi << 16), b - __uint_as_float(hi & 0xFFFF0000u)) : hi;
    }
    *reinterpret_cast<uint4*>(blk + (((j0 + q) ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// fp32 row of 32 floats (128 bytes) into a 128B-swizzled tile of [128 rows x 32 fp32] blocks
// of 16 KB: the shared-memory image of one TMA box of the fp32 output.
__device__ __forceinline__ void st_swizzled_row32_f32(uint8_t* tile, int r, int c0, const float (&v)[32],
                                                      float scale) {
  uint8_t* row = tile + (c0 >> 5) * 16384 + r * 128;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<float4*>(row + ((j ^ (r & 7)) << 4)) =
        make_float4(v[4 * j] * scale, v[4 * j + 1] * scale, v[4 * j + 2] * scale, v[4 * j + 3] * scale);
}

// S = Q K^T for one tile.  Query tile and key tile in shared memory: QB [rows x 64] SW128
// blocks of latent (or per-head key) columns, then (absorbed) the rotated positional columns: one
// [rows x d_rope] block swizzled at its row width (32, 64 or 128 bytes), or three [rows x 32] SW64
// blocks for 96 rotary dims.  Descriptors are built once and advanced by compile-time offsets.
template <class C>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t sq, uint32_t stage) {
  constexpr uint32_t idesc = C::F16 ? idesc_f16_f32(128, C::BN, false, false) : idesc_bf16_f32(128, C::BN, false, false);
  constexpr int KL = C::QB * 4;  // k-steps over the SW128 blocks
  const uint64_t kd = smem_desc(stage, 16, 1024, LAYOUT_SW128);
  const uint64_t qd = smem_desc(sq, 16, 1024, LAYOUT_SW128);
#pragma unroll
  for (int kk = 0; kk < KL; ++kk) {
    const uint64_t a = desc_add(qd, (kk >> 2) * 16384 + (kk & 3) * 32);
    const uint64_t b = desc_add(kd, (kk >> 2) * C::KBLK + (kk & 3) * 32);
    if (kk == 0)
      mma_ss_c<false>(d_tmem, a, b, idesc);
    else
      mma_ss_c<true>(d_tmem, a, b, idesc);
  }
  if constexpr (!C::DENSE) {
#pragma unroll
    for (int rb = 0; rb < C::NRB; ++rb) {
      const uint64_t krd = smem_desc(stage + C::QB * C::KBLK + rb * C::BN * C::RB, 16, 8 * C::RB, C::R_LAYOUT);
      const uint64_t qrd = smem_desc(sq + C::QB * 16384 + rb * 128 * C::RB, 16, 8 * C::RB, C::R_LAYOUT);
#pragma unroll
      for (int kk = 0; kk < C::RB / 32; ++kk)
        mma_ss_c<true>(d_tmem, desc_add(qrd, kk * 32), desc_add(krd, kk * 32), idesc);
    }
  }
}

template <class C>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t stage, bool accumulate) {
  constexpr uint32_t idesc = C::F16 ? idesc_f16_f32(128, C::DV, false, true) : idesc_bf16_f32(128, C::DV, false, true);
  const uint64_t vd = smem_desc(C::DENSE ? stage + 2 * C::KBLK : stage, C::KBLK, 1024, LAYOUT_SW128);
  if (accumulate)
    mma_ts_c<true>(o_tmem, p_tmem, vd, idesc);
  else
    mma_ts_c<false>(o_tmem, p_tmem, vd, idesc);
#pragma unroll
  for (int kk = 1; kk < C::BN / 16; ++kk) mma_ts_c<true>(o_tmem, p_tmem + kk * 8, desc_add(vd, kk * 2048), idesc);
}

template <int HS>
__device__ __forceinline__ void ld_half_tile(uint32_t taddr, uint32_t (&r)[HS]) {
  if constexpr (HS == 96) {
    tmem_ld64(taddr, *reinterpret_cast<uint32_t(*)[64]>(&r[0]));
    tmem_ld32(taddr + 64, *reinterpret_cast<uint32_t(*)[32]>(&r[64]));
  } else if constexpr (HS == 64) {
    tmem_ld64(taddr, r);
  } else if constexpr (HS == 48) {
    tmem_ld48(taddr, r);
  } else {
    tmem_ld32(taddr, r);
  }
}

template <int NP>
__device__ __forceinline__ void st_packed(uint32_t taddr, const uint32_t (&r)[NP]) {
  if constexpr (NP == 32) {
    tmem_st32(taddr, r);
  } else if constexpr (NP == 24) {
    tmem_st24(taddr, r);
  } else {
    tmem_st16(taddr, r);
  }
}

// One warp's share of an arrival: every lane has fenced its own tcgen05 traffic.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// FOLD (absorbed only): the epilogue stores O_bar itself, as its bf16 pair, for an output
// mixer that folds W_uv,h in (tm_wuv then maps O_bar's rounded part, tm_out its residual).
template <int DL, bool DENSE, bool FOLD, int DR, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kr,
                   const __grid_constant__ CUtensorMap tm_wuv, const __grid_constant__ CUtensorMap tm_out,
                   const AttnTc a) {
  using C = AttnCfg<DL, DENSE, DR, F16>;
  // The dynamic shared memory window starts 1024-byte aligned (the swizzled TMA tiles need it);
  // the whole 227 KB budget may be in use, so there is no slack to realign: check instead.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(a.err, DEV_ERR_BOUNDS);
    return;
  }
  uint8_t* sQ = smem_raw;
  uint8_t* sKV = smem_raw + C::Q_BYTES;
  Bars* bars = reinterpret_cast<Bars*>(sKV + C::STAGES * C::STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x, h = a.h0 + (int)blockIdx.y, b = blockIdx.z;
  const int m0 = mt * 128;
  const int n_tiles = (a.n_keys + C::BN - 1) / C::BN;
  const int epi_wuv = (n_tiles % C::STAGES) * C::STAGE_BYTES;           // W_uv,h
  const int epi_lo = ((n_tiles + 1) % C::STAGES) * C::STAGE_BYTES;      // O_bar residual
  const Guard g{&bars->abort_flag, a.err, a.limit_ns};

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int k = 0; k < C::NSB; ++k) {
      mbar_init(&bars->s_full[k], 1);
      mbar_init(&bars->p_full[k], kSoftmaxWarps);
      mbar_init(&bars->p_done[k], 1);
    }
    mbar_init(&bars->o_final, 1);
    mbar_init(&bars->wuv_full, 1);
    mbar_init(&bars->ob_full, kSoftmaxWarps);
    mbar_init(&bars->epi_done, 1);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->drain_pv, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tslot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tslot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_q);
      const int qrow = b * a.n_heads + h;
      mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
      for (int qb = 0; qb < C::QB; ++qb) tma_load_3d(sQ + qb * 16384, &tm_q, &bars->q_full, qb * 64, m0, qrow);
      if constexpr (!C::DENSE)
        for (int rb = 0; rb < C::NRB; ++rb)
          tma_load_3d(sQ + C::QB * 16384 + rb * 128 * C::RB, &tm_qr, &bars->q_full, DL + rb * (C::RB / 2), m0, qrow);
      int issued = 0, issued_v = 0;  // tiles (per-head: K halves) and per-head V halves in flight
      if constexpr (C::DENSE) {
        // K_t, then V_{t-1}: a K half waits behind a V half whose stage frees one tile earlier
        for (int t = 0; t <= n_tiles; ++t) {
          if (t < n_tiles) {
            const int s = t % C::STAGES;
            if (!wait_phase(&bars->kv_empty[s], ((t / C::STAGES) & 1) ^ 1, g, DEV_ERR_TIMEOUT_PRODUCER)) break;
            uint8_t* st = sKV + s * C::STAGE_BYTES;
            mbar_arrive_expect_tx(&bars->kv_full[s], 2 * C::KBLK);
            for (int kb = 0; kb < 2; ++kb)
              tma_load_3d(st + kb * C::KBLK, &tm_k, &bars->kv_full[s], h * 128 + kb * 64, t * C::BN, b);
            ++issued;
          }
          if (t > 0) {
            const int v = t - 1, s = v % C::STAGES;
            if (!wait_phase(&bars->v_empty[s], ((v / C::STAGES) & 1) ^ 1, g, DEV_ERR_TIMEOUT_PRODUCER)) break;
            uint8_t* st = sKV + s * C::STAGE_BYTES;
            mbar_arrive_expect_tx(&bars->v_full[s], 2 * C::KBLK);
            for (int kb = 0; kb < 2; ++kb)
              tma_load_3d(st + (2 + kb) * C::KBLK, &tm_k, &bars->v_full[s], (a.n_heads + h) * 128 + kb * 64,
                          v * C::BN, b);
            ++issued_v;
          }
        }
      } else {
        for (int j = 0; j < n_tiles; ++j) {
          const int s = j % C::STAGES;
          if (!wait_phase(&bars->kv_empty[s], ((j / C::STAGES) & 1) ^ 1, g, DEV_ERR_TIMEOUT_PRODUCER)) break;
          uint8_t* st = sKV + s * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&bars->kv_full[s], C::STAGE_BYTES);
          for (int kb = 0; kb < C::QB; ++kb)
            tma_load_3d(st + kb * C::KBLK, &tm_k, &bars->kv_full[s], kb * 64, j * C::BN, b);
          for (int rb = 0; rb < C::NRB; ++rb)
            tma_load_3d(st + C::QB * C::KBLK + rb * C::BN * C::RB, &tm_kr, &bars->kv_full[s], rb * (C::RB / 2),
                        j * C::BN, b);
          ++issued;
        }
      }
      bool wuv_issued = false;
      if constexpr (!C::DENSE && !FOLD) {
        // W_uv,h goes into the stage a further tile would take, as soon as P V has freed it
        const int sw = n_tiles % C::STAGES;
        if (issued == n_tiles &&
            wait_phase(&bars->kv_empty[sw], ((n_tiles / C::STAGES) & 1) ^ 1, g, DEV_ERR_TIMEOUT_PRODUCER)) {
          mbar_arrive_expect_tx(&bars->wuv_full, C::DV * 256);
          for (int kb = 0; kb < C::DV / 64; ++kb)
            tma_load_3d(sKV + epi_wuv + kb * 16384, &tm_wuv, &bars->wuv_full, kb * 64, 0, h);
          wuv_issued = true;
        }
      }
      if (bars->abort_flag) {
        drain_phase(&bars->q_full, 0, g);
        for (int j = issued > C::STAGES ? issued - C::STAGES : 0; j < issued; ++j)
          drain_phase(&bars->kv_full[j % C::STAGES], (j / C::STAGES) & 1, g);
        for (int j = issued_v > C::STAGES ? issued_v - C::STAGES : 0; j < issued_v; ++j)
          drain_phase(&bars->v_full[j % C::STAGES], (j / C::STAGES) & 1, g);
        if (wuv_issued) drain_phase(&bars->wuv_full, 0, g);
      }
    }
  } else if (warp == 1 && !C::DENSE) {
    // ------------------------------------------------------------ MMA issuer (absorbed)
    // order: QK_0 .. QK_{NSB-2}, then per tile j: QK_{j+NSB-1}, P V_j.  QK_{j+NSB-1} goes into the
    // buffer that held P_{j-1}; P V_{j-1} was issued before it, and the tensor pipe runs in order.
    if (lane == 0) {
      const uint32_t sq = smem_u32(sQ), skv = smem_u32(sKV);
      bool ok = wait_phase(&bars->q_full, 0, g, DEV_ERR_TIMEOUT_MMA);
      for (int j0 = 0; ok && j0 < C::NSB - 1 && j0 < n_tiles; ++j0) {
        const int s0 = j0 % C::STAGES;
        if (!(ok = wait_phase(&bars->kv_full[s0], (j0 / C::STAGES) & 1, g, DEV_ERR_TIMEOUT_MMA))) break;
        tc_fence_after();
        issue_qk<C>(tbase + C::S_COL + j0 * C::BN, sq, skv + s0 * C::STAGE_BYTES);
        mma_commit(&bars->s_full[j0]);
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int buf = j % C::NSB;
        const int jn = j + C::NSB - 1;
        if (jn < n_tiles) {
          const int s1 = jn % C::STAGES;
          if (!(ok = wait_phase(&bars->kv_full[s1], (jn / C::STAGES) & 1, g, DEV_ERR_TIMEOUT_MMA))) break;
          tc_fence_after();
          issue_qk<C>(tbase + C::S_COL + (jn % C::NSB) * C::BN, sq, skv + s1 * C::STAGE_BYTES);
          mma_commit(&bars->s_full[jn % C::NSB]);
        }
        if (!(ok = wait_phase(&bars->p_full[buf], (j / C::NSB) & 1, g, DEV_ERR_TIMEOUT_MMA))) break;
        tc_fence_after();
        const int s = j % C::STAGES;
        issue_pv<C>(tbase + C::O_COL, tbase + C::S_COL + buf * C::BN, skv + s * C::STAGE_BYTES, j > 0);
        mma_commit(&bars->kv_empty[s]);
        mma_commit(&bars->p_done[buf]);
      }
      if (ok) mma_commit(&bars->o_final);
      if constexpr (!C::DENSE && !FOLD) {
        // fused value up-projection: out_h = O_bar W_uv,h^T, O_bar as a bf16 pair (rounded + residual)
        if (ok && wait_phase(&bars->ob_full, 0, g, DEV_ERR_TIMEOUT_MMA) &&
            wait_phase(&bars->wuv_full, 0, g, DEV_ERR_TIMEOUT_MMA)) {
          tc_fence_after();
          constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
          const uint64_t hd = smem_desc(sq, 16, 1024, LAYOUT_SW128);
          const uint64_t ld = smem_desc(skv + epi_lo, 16, 1024, LAYOUT_SW128);
          const uint64_t wd = smem_desc(skv + epi_wuv, 16, 1024, LAYOUT_SW128);
#pragma unroll
          for (int kk = 0; kk < C::DV / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            if (kk == 0)
              mma_ss_c<false>(tbase, desc_add(hd, off), desc_add(wd, off), idesc);
            else
              mma_ss_c<true>(tbase, desc_add(hd, off), desc_add(wd, off), idesc);
            mma_ss_c<true>(tbase, desc_add(ld, off), desc_add(wd, off), idesc);
          }
          mma_commit(&bars->epi_done);
        }
      }
      if (bars->abort_flag) {
        mma_commit(&bars->drain);
        drain_phase(&bars->drain, 0, g);
      }
    }
  } else if (C::DENSE && (warp == 2 || warp == 3)) {
    // ------------------------------------------------------------ per-head MMA issuers
    // Q K^T from warp 2 and P V from warp 3 (one thread each, on SM sub-partitions of their own), so
    // neither stream of MMAs waits behind the other's issue.  Ordering between them is by barriers:
    // Q K_t^T overwrites the S buffer of P_{t-NSB} only once P V_{t-NSB} has completed.
    if (lane == 0) {
      const uint32_t sq = smem_u32(sQ), skv = smem_u32(sKV);
      bool ok = true;
      if (warp == 2) {
        ok = wait_phase(&bars->q_full, 0, g, DEV_ERR_TIMEOUT_MMA);
        for (int t = 0; ok && t < n_tiles; ++t) {
          const int sb = t % C::NSB, s = t % C::STAGES;
          if (t >= C::NSB &&
              !(ok = wait_phase(&bars->p_done[sb], ((t - C::NSB) / C::NSB) & 1, g, DEV_ERR_TIMEOUT_MMA)))
            break;
          if (!(ok = wait_phase(&bars->kv_full[s], (t / C::STAGES) & 1, g, DEV_ERR_TIMEOUT_MMA))) break;
          tc_fence_after();
          issue_qk<C>(tbase + C::S_COL + sb * C::BN, sq, skv + s * C::STAGE_BYTES);
          mma_commit(&bars->kv_empty[s]);
          mma_commit(&bars->s_full[sb]);
        }
        if (bars->abort_flag) {
          mma_commit(&bars->drain);
          drain_phase(&bars->drain, 0, g);
        }
      } else {
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int sb = j % C::NSB, s = j % C::STAGES;
          if (!(ok = wait_phase(&bars->p_full[sb], (j / C::NSB) & 1, g, DEV_ERR_TIMEOUT_MMA))) break;
          if (!(ok = wait_phase(&bars->v_full[s], (j / C::STAGES) & 1, g, DEV_ERR_TIMEOUT_MMA))) break;
          tc_fence_after();
          issue_pv<C>(tbase + C::O_COL, tbase + C::S_COL + sb * C::BN, skv + s * C::STAGE_BYTES, j > 0);
          mma_commit(&bars->v_empty[s]);
          mma_commit(&bars->p_done[sb]);
        }
        if (ok) mma_commit(&bars->o_final);
        if (bars->abort_flag) {
          mma_commit(&bars->drain_pv);
          drain_phase(&bars->drain_pv, 0, g);
        }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax / correction / epilogue
    // Two warpgroups share the 128 rows: group wg takes score columns [wg*BN/2, (wg+1)*BN/2)
    // of every tile and O columns [wg*DV/2, (wg+1)*DV/2); warp w of either group reads TMEM
    // lanes 32*(w%4).. (the same rows).  The row max of a tile is the larger of the two
    // halves' maxima, swapped through shared memory once per tile by the two warps of a lane
    // quarter alone (named barrier 2 + quarter, 64 threads).  Every thread of both groups
    // passes the same named barriers in the same order, whatever happens: a thread that gave
    // up skips the work, never the barrier.
    const int wg = (warp - 4) >> 2;
    const int wq = (warp - 4) & 3;
    const int r = wq * 32 + lane;  // query row inside the tile == TMEM lane
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(wq * 32) << 16);
    constexpr int HS = C::BN / 2;  // score columns per group
    constexpr int HO = C::DV / 2;  // O columns per group
    const int sc0 = wg * HS;
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int buf = j % C::NSB;  // S buffer of tile j
      const int xp = j & 1;        // exchange slot of tile j
      ok = ok && __all_sync(0xffffffffu, wait_phase(&bars->s_full[buf], (j / C::NSB) & 1, g, DEV_ERR_TIMEOUT_SOFTMAX));
      uint32_t sraw[HS];
      float mx = -INFINITY;
      if (ok) {
        tc_fence_after();
        ld_half_tile<HS>(lane_base + C::S_COL + buf * C::BN + sc0, sraw);
        const int valid = a.n_keys - j * C::BN - sc0;
        if (valid < HS) {  // only the last tile is ragged (warp-uniform branch)
#pragma unroll
          for (int c = 0; c < HS; ++c)
            if (c >= valid) sraw[c] = __float_as_uint(-INFINITY);
        }
        // half-row max: independent chains of 3-input max over 16 scores each
        float mxc[HS / 16];
#pragma unroll
        for (int k = 0; k < HS / 16; ++k) {
          const uint32_t* v = &sraw[16 * k];
          float m = max3f(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
          for (int i = 3; i < 15; i += 2) m = max3f(m, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
          mxc[k] = fmaxf(m, __uint_as_float(v[15]));
        }
        mx = mxc[0];
#pragma unroll
        for (int k = 1; k < HS / 16; ++k) mx = fmaxf(mx, mxc[k]);
      }
      bars->red[xp][wg][r] = mx;
      named_bar_sync(2 + wq, 64);  // the two warps of this lane quarter (one per group) exchange
      const float m_tile = fmaxf(mx, bars->red[xp][wg ^ 1][r]) * a.scale_log2;
      if (ok) {
        if (j == 0) {
          m_run = m_tile;
        } else if (__any_sync(0xffffffffu, m_tile > m_run + a.rescale_threshold)) {
          // raise the running max of every row of this warp; rescale this group's half of O
          // once the previous P V is done (both groups take the same decision for a row)
          const float m_new = fmaxf(m_run, m_tile);
          const float alpha = ex2_approx(m_run - m_new);
          ok = __all_sync(0xffffffffu, wait_phase(&bars->p_done[(j - 1) % C::NSB], ((j - 1) / C::NSB) & 1, g,
                                                  DEV_ERR_TIMEOUT_SOFTMAX));
          if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int c = wg * HO; c < (wg + 1) * HO; c += 32) {
              uint32_t o[32];
              tmem_ld32(lane_base + C::O_COL + c, o);
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st32(lane_base + C::O_COL + c, o);
            }
            l_run *= alpha;
            m_run = m_new;
          }
        }
      }
      if (ok) {
        // p = 2^(s*scale - m): scale-and-subtract two scores per instruction, exp2 on the MUFU,
        // row sum in four independent packed accumulators, bf16 pairs back into TMEM over S
        const float2 nm2 = make_float2(-m_run, -m_run);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        if constexpr (HS % 32 == 0 && HS > 64) {
          // wide tiles: P leaves in 16-column pieces as it is made, so the pieces' registers recycle
#pragma unroll
          for (int c = 0; c < HS / 32; ++c) {
            uint32_t packed[16];
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) {
              const int k = 16 * c + kk;
              const float2 x = make_float2(__uint_as_float(sraw[2 * k]), __uint_as_float(sraw[2 * k + 1]));
              const float2 y = __ffma2_rn(x, sc2, nm2);
              const float2 pr = exp2_mixed(y, k);
              acc[k & 3] = __fadd2_rn(acc[k & 3], pr);
              packed[kk] = C::F16 ? pack_f16x2(pr.x, pr.y) : pack_bf16x2(pr.x, pr.y);
            }
            tmem_st16_async(lane_base + C::S_COL + buf * C::BN + wg * (HS / 2) + 16 * c, packed);
          }
          tmem_wait_st();
        } else {
          uint32_t packed[HS / 2];
#pragma unroll
          for (int k = 0; k < HS / 2; ++k) {
            const float2 x = make_float2(__uint_as_float(sraw[2 * k]), __uint_as_float(sraw[2 * k + 1]));
            const float2 y = __ffma2_rn(x, sc2, nm2);
            const float2 pr = exp2_mixed(y, k);
            acc[k & 3] = __fadd2_rn(acc[k & 3], pr);
            packed[k] = C::F16 ? pack_f16x2(pr.x, pr.y) : pack_bf16x2(pr.x, pr.y);
          }
          st_packed<HS / 2>(lane_base + C::S_COL + buf * C::BN + wg * (HS / 2), packed);
        }
        const float2 acc4 = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
        l_run += acc4.x + acc4.y;
        tc_fence_before();
      }
      warp_arrive(&bars->p_full[buf]);
    }
    ok = ok && __all_sync(0xffffffffu, wait_phase(&bars->o_final, 0, g, DEV_ERR_TIMEOUT_EPILOGUE));
    if (ok) tc_fence_after();
    // row sum = both halves' partial sums (the other parity's exchange slot is free by now)
    bars->red[n_tiles & 1][wg][r] = l_run;
    named_bar_sync(2 + wq, 64);
    const float inv_l = 1.f / (l_run + bars->red[n_tiles & 1][wg ^ 1][r]);
    if constexpr (!C::DENSE) {
      // O_bar = O / l as a bf16 pair (A operands of the two W_uv GEMMs): rounded part over the
      // query tile, residual in the ring stage after W_uv,h's
      if (ok) {
#pragma unroll 1
        for (int c = wg * HO; c < (wg + 1) * HO; c += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + C::O_COL + c, o);
          st_swizzled_row32(sQ, r, c, *reinterpret_cast<float(*)[32]>(o), inv_l, false);
          st_swizzled_row32(sKV + epi_lo, r, c, *reinterpret_cast<float(*)[32]>(o), inv_l, true);
        }
      }
      fence_async_smem();
      tc_fence_before();
      if constexpr (FOLD) {
        named_bar_sync(1, 256);
        if (wg == 0 && r == 0 && ok && !bars->abort_flag) {
          for (int blk = 0; blk < C::DV / 64; ++blk) {
            tma_store_3d(&tm_wuv, sQ + blk * 16384, h * DL + blk * 64, m0, b);
            tma_store_3d(&tm_out, sKV + epi_lo + blk * 16384, h * DL + blk * 64, m0, b);
          }
          bulk_commit();
          bulk_wait_all_read();
        }
      } else {
      warp_arrive(&bars->ob_full);
      ok = ok && __all_sync(0xffffffffu, wait_phase(&bars->epi_done, 0, g, DEV_ERR_TIMEOUT_EPILOGUE));
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c = wg * 64; c < wg * 64 + 64; c += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + c, o);
          st_swizzled_row32_f32(sKV, r, c, *reinterpret_cast<float(*)[32]>(o), 1.f);
        }
      }
      }
    } else {
      if (ok) {
#pragma unroll 1
        for (int c = wg * 64; c < wg * 64 + 64; c += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + C::O_COL + c, o);
          st_swizzled_row32_f32(sKV, r, c, *reinterpret_cast<float(*)[32]>(o), inv_l);
        }
      }
    }
    if constexpr (!FOLD) {
      fence_async_smem();
      named_bar_sync(1, 256);
      if (wg == 0 && r == 0 && !bars->abort_flag) {
        for (int blk = 0; blk < 4; ++blk) tma_store_3d(&tm_out, sKV + blk * 16384, h * 128 + blk * 32, m0, b);
        bulk_commit();
        bulk_wait_all_read();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

template <int DL, bool DENSE, bool FOLD = false, int DR = 32, bool F16 = false>
cudaError_t go_attn(const CUtensorMap& tq, const CUtensorMap& tqr, const CUtensorMap& tk, const CUtensorMap& tkr,
                    const CUtensorMap& tuv, const CUtensorMap& to, const AttnTc& a, int batch, cudaStream_t s) {
  using C = AttnCfg<DL, DENSE, DR, F16>;
  static const cudaError_t attr = cudaFuncSetAttribute(attn_tc_kernel<DL, DENSE, FOLD, DR, F16>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (attr != cudaSuccess) return attr;
  if (a.n_q <= 0 || a.n_keys <= 0) return cudaSuccess;
  const int heads = a.h_count > 0 ? a.h_count : a.n_heads;
  attn_tc_kernel<DL, DENSE, FOLD, DR, F16><<<dim3(a.m_tiles, heads, batch), kThreads, C::SMEM, s>>>(
      tq, tqr, tk, tkr, tuv, to, a);
  return cudaGetLastError();
}

}  // namespace

int attn_absorbed_block_n(int d_latent) {
  switch (d_latent) {
    case 64: return AttnCfg<64, false>::BN;
    case 128: return AttnCfg<128, false>::BN;
    case 192: return AttnCfg<192, false>::BN;
    case 256: return AttnCfg<256, false>::BN;
  }
  return 128;
}

int attn_dense_block_n() { return AttnCfg<128, true>::BN; }

template <int DR>
cudaError_t go_attn_obar_dl(int d_latent, const CUtensorMap& tq, const CUtensorMap& tqr, const CUtensorMap& tk,
                            const CUtensorMap& tkr, const CUtensorMap& tob_hi, const CUtensorMap& tob_lo,
                            const AttnTc& a, int batch, cudaStream_t s) {
  switch (d_latent) {
    case 64: return go_attn<64, false, true, DR>(tq, tqr, tk, tkr, tob_hi, tob_lo, a, batch, s);
    case 128: return go_attn<128, false, true, DR>(tq, tqr, tk, tkr, tob_hi, tob_lo, a, batch, s);
    case 192: return go_attn<192, false, true, DR>(tq, tqr, tk, tkr, tob_hi, tob_lo, a, batch, s);
    case 256:
      if constexpr (DR <= 32) return go_attn<256, false, true, DR>(tq, tqr, tk, tkr, tob_hi, tob_lo, a, batch, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_absorbed_obar_tc(int d_latent, int d_rope, const CUtensorMap& tq, const CUtensorMap& tqr,
                                         const CUtensorMap& tk, const CUtensorMap& tkr, const CUtensorMap& tob_hi,
                                         const CUtensorMap& tob_lo, const AttnTc& a, int batch, cudaStream_t s) {
  switch (d_rope) {
    case 16: return go_attn_obar_dl<16>(d_latent, tq, tqr, tk, tkr, tob_hi, tob_lo, a, batch, s);
    case 32: return go_attn_obar_dl<32>(d_latent, tq, tqr, tk, tkr, tob_hi, tob_lo, a, batch, s);
    case 64: return go_attn_obar_dl<64>(d_latent, tq, tqr, tk, tkr, tob_hi, tob_lo, a, batch, s);
    case 96: return go_attn_obar_dl<96>(d_latent, tq, tqr, tk, tkr, tob_hi, tob_lo, a, batch, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_dense_tc(const CUtensorMap& tq, const CUtensorMap& tkv, const CUtensorMap& to,
                                 const AttnTc& a, int batch, cudaStream_t s, bool f16) {
  if (f16) return go_attn<128, true, false, 32, true>(tq, tq, tkv, tkv, tq, to, a, batch, s);
  return go_attn<128, true>(tq, tq, tkv, tkv, tq, to, a, batch, s);
}

bool attn_absorbed_supported(int d_latent, int d_rope) {
  const bool dl = d_latent == 64 || d_latent == 128 || d_latent == 192 || d_latent == 256;
  return dl && (d_rope == 16 || d_rope == 32 || ((d_rope == 64 || d_rope == 96) && d_latent <= 192));
}

template <int DR>
cudaError_t go_attn_dl(int d_latent, const CUtensorMap& tq, const CUtensorMap& tqr, const CUtensorMap& tk,
                       const CUtensorMap& tkr, const CUtensorMap& tuv, const CUtensorMap& to, const AttnTc& a,
                       int batch, cudaStream_t s) {
  switch (d_latent) {
    case 64: return go_attn<64, false, false, DR>(tq, tqr, tk, tkr, tuv, to, a, batch, s);
    case 128: return go_attn<128, false, false, DR>(tq, tqr, tk, tkr, tuv, to, a, batch, s);
    case 192: return go_attn<192, false, false, DR>(tq, tqr, tk, tkr, tuv, to, a, batch, s);
    case 256:
      if constexpr (DR <= 32) return go_attn<256, false, false, DR>(tq, tqr, tk, tkr, tuv, to, a, batch, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_absorbed_tc(int d_latent, int d_rope, const CUtensorMap& tq, const CUtensorMap& tqr,
                                    const CUtensorMap& tk, const CUtensorMap& tkr, const CUtensorMap& tuv,
                                    const CUtensorMap& to, const AttnTc& a, int batch, cudaStream_t s) {
  switch (d_rope) {
    case 16: return go_attn_dl<16>(d_latent, tq, tqr, tk, tkr, tuv, to, a, batch, s);
    case 32: return go_attn_dl<32>(d_latent, tq, tqr, tk, tkr, tuv, to, a, batch, s);
    case 64: return go_attn_dl<64>(d_latent, tq, tqr, tk, tkr, tuv, to, a, batch, s);
    case 96: return go_attn_dl<96>(d_latent, tq, tqr, tk, tkr, tuv, to, a, batch, s);
  }
  return cudaErrorInvalidValue;
}


}  // namespace vmla
