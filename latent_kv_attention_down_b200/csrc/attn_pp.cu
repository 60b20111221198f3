// Per-head chunk attention with two query tiles per CTA taking turns on the tensor core
// (sm_100a): the d_head = 128 attention of the reconstruct-once design (fp16 operands) and of
// the dense per-head comparison (bf16), out_h = softmax(q_h K_h^T / sqrt(d_head)) V_h
// [paperlayer §3 "On-demand reconstruction"].
//
// One CTA holds query tiles A and B (128 rows each, the same head) and streams the head's
// keys once for both:
//   warp 0      TMA producer: the two query tiles per segment, then K_j and V_j tiles (32 KB
//               each) into a ring of five slots
//   warp 1      tcgen05.mma issuer (one thread) + TMEM owner
//   warps 4-7   softmax of tile A, warps 8-11 softmax of tile B: thread r owns query row r
//               (TMEM lane r) and all 128 scores of a key tile, so the row max needs no
//               exchange between warps
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512); P_X is written
// as fp16 (or bf16) pairs over the first 64 columns of S_X and read from there by P V.
// The tensor core alternates between the tiles: P_A V_j and Q_A K_{j+1}^T run while the
// softmax of B works on S_B(j), then P_B V_j and Q_B K_{j+1}^T while the softmax of A works
// on S_A(j+1), so MMA and exponentials overlap instead of waiting on each other.
//
// Work split (stream-K): the (tile pair, key tile) iterations of all pairs of the launch are
// cut into `ctas` equal contiguous ranges, one per CTA.  A CTA therefore runs a few segments
// (a key range of one pair); a pair whose keys span several CTAs leaves a partial (O unscaled,
// running max m and sum l per row) from each, and attn_pp_merge_kernel combines them.  A
// segment covering all keys writes its rows normalised.  The last pair of a (sample, head)
// with an odd number of query tiles runs tile A alone.
// The running max is only raised when it grows by more than 2^threshold (lazy rescale);
// O_X is then rescaled in TMEM once P V of the previous tile has finished.  Every mbarrier
// wait is bounded; a CTA that gives up records the error and drains its copies and MMAs
// before releasing TMEM.
#include "kernels.h"
#include "ptx.cuh"

namespace vmla {
namespace {

constexpr int kPPThreads = 384;
constexpr int kPPSlots = 5;
constexpr int kPPTile = 32768;  // one 128 x 128 fp16/bf16 tile: two [128 x 64] SW128 blocks

struct PPBars {
  uint64_t q_full, q_empty;
  uint64_t kv_full[kPPSlots], kv_empty[kPPSlots];
  uint64_t s_full[2], p_full[2], pv_done[2];  // per query tile (A, B)
  uint64_t o_full[2];                         // every MMA of the segment done
  uint64_t epi_done[2];                       // the tile's epilogue has read O
  uint64_t drain;
  uint32_t tslot;
  int abort_flag;
};

constexpr int kPPBars = (sizeof(PPBars) + 127) / 128 * 128;
constexpr int kPPSmem = 2 * kPPTile + kPPSlots * kPPTile + kPPBars;
static_assert(kPPSmem <= 232448, "shared memory budget");

// One segment of a CTA's iteration range: pair p over key tiles [k0, k1).
struct Seg {
  int p, k0, k1;
  int b, h, tile_a;
  bool two;    // tile B = tile_a + 1 exists
  bool whole;  // every key of the pair: rows are written normalised
  int slot;    // partial slot (when !whole)
};

__device__ __forceinline__ int64_t pp_it0(const AttnPP& a, int g) { return a.iters * g / a.ctas; }

__device__ __forceinline__ Seg pp_seg(const AttnPP& a, int g, int64_t it, int64_t it1) {
  Seg s;
  s.p = (int)(it / a.n_kt);
  s.k0 = (int)(it - (int64_t)s.p * a.n_kt);
  const int64_t rest = it1 - it;
  s.k1 = rest < (int64_t)(a.n_kt - s.k0) ? s.k0 + (int)rest : a.n_kt;
  const int bh = s.p / a.pairs_per_bh, pi = s.p - bh * a.pairs_per_bh;
  s.b = bh / a.h_count;
  s.h = a.h0 + (bh - s.b * a.h_count);
  s.tile_a = 2 * pi;
  s.two = s.tile_a + 1 < a.m_tiles;
  s.whole = s.k0 == 0 && s.k1 == a.n_kt;
  s.slot = 2 * g + (s.p == (int)(pp_it0(a, g) / a.n_kt) ? 0 : 1);
  return s;
}

// S_X = Q_X K_j^T: Q and K tiles as two [128 x 64] SW128 blocks, K-major.
template <bool F16>
__device__ __forceinline__ void pp_qk(uint32_t d_tmem, uint32_t sq, uint32_t sk) {
  constexpr uint32_t idesc = F16 ? idesc_f16_f32(128, 128, false, false) : idesc_bf16_f32(128, 128, false, false);
  const uint64_t qd = smem_desc(sq, 16, 1024, LAYOUT_SW128);
  const uint64_t kd = smem_desc(sk, 16, 1024, LAYOUT_SW128);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
    if (kk == 0)
      mma_ss_c<false>(d_tmem, desc_add(qd, off), desc_add(kd, off), idesc);
    else
      mma_ss_c<true>(d_tmem, desc_add(qd, off), desc_add(kd, off), idesc);
  }
}

// O_X (+)= P_X V_j: P from TMEM (8 columns per 16 keys), V as the MN-major B operand.
template <bool F16>
__device__ __forceinline__ void pp_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t sv, bool accumulate) {
  constexpr uint32_t idesc = F16 ? idesc_f16_f32(128, 128, false, true) : idesc_bf16_f32(128, 128, false, true);
  const uint64_t vd = smem_desc(sv, 16384, 1024, LAYOUT_SW128);
  if (accumulate)
    mma_ts_c<true>(o_tmem, p_tmem, vd, idesc);
  else
    mma_ts_c<false>(o_tmem, p_tmem, vd, idesc);
#pragma unroll
  for (int kk = 1; kk < 8; ++kk) mma_ts_c<true>(o_tmem, p_tmem + kk * 8, desc_add(vd, kk * 2048), idesc);
}

__device__ __forceinline__ void pp_warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// TMEM columns of S_X and O_X for tile x (0: A, 1: B)
__device__ __forceinline__ uint32_t s_col_of(int x) { return 128u * x; }
__device__ __forceinline__ uint32_t o_col_of(int x) { return 256u + 128u * x; }

template <bool F16>
__global__ void __launch_bounds__(kPPThreads, 1)
    attn_pp_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                   const AttnPP a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(a.err, DEV_ERR_BOUNDS);
    return;
  }
  uint8_t* sQ = smem_raw;                   // Q_A at 0, Q_B at kPPTile
  uint8_t* sKV = smem_raw + 2 * kPPTile;    // ring slots
  PPBars* bars = reinterpret_cast<PPBars*>(sKV + kPPSlots * kPPTile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x;
  const int64_t it_begin = pp_it0(a, g), it_end = pp_it0(a, g + 1);
  const Guard gd{&bars->abort_flag, a.err, a.limit_ns};

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kPPSlots; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_full[x], 4);
      mbar_init(&bars->pv_done[x], 1);
      mbar_init(&bars->o_full[x], 1);
      mbar_init(&bars->epi_done[x], 4);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tslot;
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_kv);
      int q_issued = 0, n_seg = 0;
      int64_t slot_it = 0;  // ring slot uses so far (K and V tiles alike)
      bool ok = true;
      for (int64_t it = it_begin; ok && it < it_end; ++n_seg) {
        const Seg s = pp_seg(a, g, it, it_end);
        it += s.k1 - s.k0;
        if (n_seg > 0 && !(ok = wait_phase(&bars->q_empty, (n_seg - 1) & 1, gd, DEV_ERR_TIMEOUT_PRODUCER))) break;
        const int qrow = s.b * a.n_heads + s.h;
        mbar_arrive_expect_tx(&bars->q_full, s.two ? 2 * kPPTile : kPPTile);
        for (int t = 0; t < (s.two ? 2 : 1); ++t)
          for (int kb = 0; kb < 2; ++kb)
            tma_load_3d(sQ + t * kPPTile + kb * 16384, &tm_q, &bars->q_full, kb * 64, (s.tile_a + t) * 128, qrow);
        ++q_issued;
        for (int j = s.k0; ok && j < s.k1; ++j) {
          for (int kv = 0; kv < 2; ++kv, ++slot_it) {  // K_j, then V_j
            const int sl = (int)(slot_it % kPPSlots);
            if (!(ok = wait_phase(&bars->kv_empty[sl], (int)((slot_it / kPPSlots) & 1) ^ 1, gd,
                                  DEV_ERR_TIMEOUT_PRODUCER)))
              break;
            uint8_t* dst = sKV + sl * kPPTile;
            mbar_arrive_expect_tx(&bars->kv_full[sl], kPPTile);
            const int col = (kv * a.n_heads + s.h) * 128;
            for (int kb = 0; kb < 2; ++kb)
              tma_load_3d(dst + kb * 16384, &tm_kv, &bars->kv_full[sl], col + kb * 64, j * 128, s.b);
          }
        }
      }
      if (bars->abort_flag) {  // let the copies in flight land before the CTA goes away
        if (q_issued > 0) drain_phase(&bars->q_full, (q_issued - 1) & 1, gd);
        for (int64_t i = slot_it > kPPSlots ? slot_it - kPPSlots : 0; i < slot_it; ++i)
          drain_phase(&bars->kv_full[i % kPPSlots], (int)((i / kPPSlots) & 1), gd);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t sq = smem_u32(sQ), skv = smem_u32(sKV);
      int n_seg = 0, n_epi[2] = {0, 0}, n_tiles[2] = {0, 0};
      int64_t slot_it = 0;
      bool ok = true;
      auto take = [&](int64_t use) -> uint32_t {  // wait for ring use `use`, return its address
        const int sl = (int)(use % kPPSlots);
        ok = ok && wait_phase(&bars->kv_full[sl], (int)((use / kPPSlots) & 1), gd, DEV_ERR_TIMEOUT_MMA);
        tc_fence_after();
        return skv + sl * kPPTile;
      };
      for (int64_t it = it_begin; ok && it < it_end; ++n_seg) {
        const Seg s = pp_seg(a, g, it, it_end);
        it += s.k1 - s.k0;
        const int nx = s.two ? 2 : 1;
        if (!(ok = wait_phase(&bars->q_full, n_seg & 1, gd, DEV_ERR_TIMEOUT_MMA))) break;
        tc_fence_after();
        // S_X(k0) for both tiles
        int64_t k_use = slot_it++;
        uint32_t sk = take(k_use);
        if (!ok) break;
        for (int x = 0; x < nx; ++x) {
          pp_qk<F16>(tbase + s_col_of(x), sq + x * kPPTile, sk);
          mma_commit(&bars->s_full[x]);
        }
        mma_commit(&bars->kv_empty[k_use % kPPSlots]);
        for (int j = s.k0; ok && j < s.k1; ++j) {
          const int64_t v_use = slot_it++;
          const uint32_t sv = take(v_use);
          const bool more = j + 1 < s.k1;
          int64_t kn_use = -1;
          uint32_t skn = 0;
          for (int x = 0; ok && x < nx; ++x) {
            // O_X of the previous segment must have been read out before P V overwrites it
            if (j == s.k0 && n_epi[x] > 0 &&
                !(ok = wait_phase(&bars->epi_done[x], (n_epi[x] - 1) & 1, gd, DEV_ERR_TIMEOUT_MMA)))
              break;
            if (!(ok = wait_phase(&bars->p_full[x], n_tiles[x] & 1, gd, DEV_ERR_TIMEOUT_MMA))) break;
            tc_fence_after();
            pp_pv<F16>(tbase + o_col_of(x), tbase + s_col_of(x), sv, j > s.k0);
            mma_commit(&bars->pv_done[x]);
            ++n_tiles[x];
            if (x == nx - 1) mma_commit(&bars->kv_empty[v_use % kPPSlots]);
            if (more) {
              if (x == 0) {
                kn_use = slot_it++;
                skn = take(kn_use);
                if (!ok) break;
              }
              pp_qk<F16>(tbase + s_col_of(x), sq + x * kPPTile, skn);  // S_X(j+1) over P_X(j): P V_j read it first
              mma_commit(&bars->s_full[x]);
              if (x == nx - 1) mma_commit(&bars->kv_empty[kn_use % kPPSlots]);
            }
          }
        }
        if (!ok) break;
        for (int x = 0; x < nx; ++x) {
          mma_commit(&bars->o_full[x]);
          ++n_epi[x];
        }
        mma_commit(&bars->q_empty);
      }
      if (bars->abort_flag) {
        mma_commit(&bars->drain);
        drain_phase(&bars->drain, 0, gd);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue of tile X
    const int x = (warp - 4) >> 2;
    const int wq = (warp - 4) & 3;
    const int r = wq * 32 + lane;  // query row inside the tile == TMEM lane
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_col = lane_base + s_col_of(x), o_col = lane_base + o_col_of(x);
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
    const int row_stride = a.n_heads * 128;
    int n_tiles = 0, n_seg_x = 0;
    bool ok = true;
    for (int64_t it = it_begin; ok && it < it_end;) {
      const Seg s = pp_seg(a, g, it, it_end);
      it += s.k1 - s.k0;
      if (x == 1 && !s.two) continue;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = s.k0; j < s.k1; ++j) {
        ok = __all_sync(0xffffffffu, wait_phase(&bars->s_full[x], n_tiles & 1, gd, DEV_ERR_TIMEOUT_SOFTMAX));
        if (!ok) break;
        tc_fence_after();
        // row max over the two 64-column halves (the second half stays in registers)
        uint32_t sraw[64];
        float mx = -INFINITY;
        const int valid = a.n_keys - j * 128;  // only the last key tile is ragged (warp-uniform)
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
          tmem_ld64(s_col + 64 * hf, sraw);
          if (valid < 128) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (64 * hf + c >= valid) sraw[c] = __float_as_uint(-INFINITY);
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
          mx = max3f(mx, fmaxf(mxc[0], mxc[1]), fmaxf(mxc[2], mxc[3]));
        }
        const float m_tile = mx * a.scale_log2;
        if (j == s.k0) {
          m_run = m_tile;
        } else if (__any_sync(0xffffffffu, m_tile > m_run + a.rescale_threshold)) {
          // raise the running max of every row of this warp; rescale its rows of O_X once the
          // previous P V is done
          const float m_new = fmaxf(m_run, m_tile);
          const float alpha = ex2_approx(m_run - m_new);
          ok = __all_sync(0xffffffffu,
                          wait_phase(&bars->pv_done[x], (n_tiles - 1) & 1, gd, DEV_ERR_TIMEOUT_SOFTMAX));
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 128; c += 32) {
            uint32_t o[32];
            tmem_ld32(o_col + c, o);
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(o_col + c, o);
          }
          l_run *= alpha;
          m_run = m_new;
        }
        // p = 2^(s*scale - m) two scores per instruction, exp2 on the MUFU, row sum in four
        // packed accumulators, fp16/bf16 pairs back into TMEM over S_X: the second half of the
        // scores (still in registers) first, then the first half, read again
        const float2 nm2 = make_float2(-m_run, -m_run);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll 1
        for (int hf = 1; hf >= 0; --hf) {
          if (hf == 0) {
            tmem_ld64(s_col, sraw);
            if (valid < 64) {
#pragma unroll
              for (int c = 0; c < 64; ++c)
                if (c >= valid) sraw[c] = __float_as_uint(-INFINITY);
            }
          }
          uint32_t packed[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float2 xx = make_float2(__uint_as_float(sraw[2 * k]), __uint_as_float(sraw[2 * k + 1]));
            const float2 y = __ffma2_rn(xx, sc2, nm2);
            const float2 pr = exp2_mixed(y, k);
            acc[k & 3] = __fadd2_rn(acc[k & 3], pr);
            packed[k] = F16 ? pack_f16x2(pr.x, pr.y) : pack_bf16x2(pr.x, pr.y);
          }
          tmem_st32(s_col + 32 * hf, packed);
        }
        const float2 acc4 = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
        l_run += acc4.x + acc4.y;
        tc_fence_before();
        pp_warp_arrive(&bars->p_full[x]);
        ++n_tiles;
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, wait_phase(&bars->o_full[x], n_seg_x & 1, gd, DEV_ERR_TIMEOUT_EPILOGUE));
      if (!ok) break;
      tc_fence_after();
      const int row = (s.tile_a + x) * 128 + r;
      if (s.whole) {
        const float inv_l = 1.f / l_run;
        float* dst = a.out + ((int64_t)s.b * a.n_q + row) * row_stride + s.h * 128;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t o[32];
          tmem_ld32(o_col + c, o);
          if (row < a.n_q) {
#pragma unroll
            for (int k = 0; k < 32; k += 4)
              *reinterpret_cast<float4*>(dst + c + k) =
                  make_float4(__uint_as_float(o[k]) * inv_l, __uint_as_float(o[k + 1]) * inv_l,
                              __uint_as_float(o[k + 2]) * inv_l, __uint_as_float(o[k + 3]) * inv_l);
          }
        }
      } else {
        const int64_t prow = ((int64_t)s.slot * 2 + x) * 128 + r;
        float* dst = a.part + prow * 128;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t o[32];
          tmem_ld32(o_col + c, o);
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(dst + c + k) = make_float4(__uint_as_float(o[k]), __uint_as_float(o[k + 1]),
                                                                  __uint_as_float(o[k + 2]), __uint_as_float(o[k + 3]));
        }
        *reinterpret_cast<float2*>(a.part_ml + prow * 2) = make_float2(m_run, l_run);
      }
      tc_fence_before();
      pp_warp_arrive(&bars->epi_done[x]);
      ++n_seg_x;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// Combines the partials of every pair whose keys were split between CTAs.  Block (g, x): the
// pair that starts before CTA g's first iteration and continues into it, when g is the first
// CTA boundary inside that pair; tile x of it.  Warp w takes rows w, w+4, ...; lane l columns
// 4l..4l+3.
__global__ void __launch_bounds__(128) attn_pp_merge_kernel(const AttnPP a) {
  const int g = blockIdx.x, x = blockIdx.y;
  if (g == 0 || g >= a.ctas) return;
  const int64_t b0 = pp_it0(a, g);
  if (b0 % a.n_kt == 0) return;  // the boundary falls between pairs
  const int p = (int)(b0 / a.n_kt);
  const int64_t p_begin = (int64_t)p * a.n_kt, p_end = p_begin + a.n_kt;
  if (pp_it0(a, g - 1) > p_begin) return;  // an earlier boundary inside the same pair merges it
  const Seg s = pp_seg(a, g - 1, p_begin, p_end);
  if (x == 1 && !s.two) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_stride = a.n_heads * 128;
  const int p_first = (int)(pp_it0(a, g - 1) / a.n_kt);  // every later contributor starts inside pair p
  for (int r = warp; r < 128; r += 4) {
    const int row = (s.tile_a + x) * 128 + r;
    if (row >= a.n_q) break;
    // the contributors: CTAs g-1, g, ... while their ranges start before the pair ends; CTA c's
    // piece sits in its first partial slot when p is the first pair of its range
    float m = -INFINITY;
    for (int c = g - 1; c < a.ctas && pp_it0(a, c) < p_end; ++c) {
      const int slot = 2 * c + (c == g - 1 && p != p_first ? 1 : 0);
      m = fmaxf(m, a.part_ml[(((int64_t)slot * 2 + x) * 128 + r) * 2]);
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float l = 0.f;
    for (int c = g - 1; c < a.ctas && pp_it0(a, c) < p_end; ++c) {
      const int slot = 2 * c + (c == g - 1 && p != p_first ? 1 : 0);
      const int64_t prow = ((int64_t)slot * 2 + x) * 128 + r;
      const float2 ml = *reinterpret_cast<const float2*>(a.part_ml + prow * 2);
      const float w = ex2_approx(ml.x - m);
      const float4 o = *reinterpret_cast<const float4*>(a.part + prow * 128 + 4 * lane);
      acc.x += w * o.x;
      acc.y += w * o.y;
      acc.z += w * o.z;
      acc.w += w * o.w;
      l += w * ml.y;
    }
    const float inv_l = 1.f / l;
    *reinterpret_cast<float4*>(a.out + ((int64_t)s.b * a.n_q + row) * row_stride + s.h * 128 + 4 * lane) =
        make_float4(acc.x * inv_l, acc.y * inv_l, acc.z * inv_l, acc.w * inv_l);
  }
}

}  // namespace

AttnPP attn_pp_plan(AttnPP a, int batch, int sms) {
  const int hc = a.h_count > 0 ? a.h_count : a.n_heads;
  a.h_count = hc;
  a.pairs_per_bh = (a.m_tiles + 1) / 2;
  a.n_kt = (a.n_keys + 127) / 128;
  const int64_t pairs = (int64_t)batch * hc * a.pairs_per_bh;
  a.iters = pairs * a.n_kt;
  // at least four key tiles per CTA: a segment's query load and epilogue cost about one tile
  const int64_t by_work = (a.iters + 3) / 4;
  a.ctas = (int)std::max<int64_t>(1, std::min<int64_t>(std::min(sms, kAttnPPMaxCtas), by_work));
  return a;
}

cudaError_t launch_attn_pp(const CUtensorMap& tq, const CUtensorMap& tkv, const AttnPP& a, cudaStream_t s, bool f16) {
  if (a.n_q <= 0 || a.n_keys <= 0 || a.iters <= 0) return cudaSuccess;
  if (a.ctas > kAttnPPMaxCtas) return cudaErrorInvalidValue;
  static const cudaError_t attr16 =
      cudaFuncSetAttribute(attn_pp_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPPSmem);
  static const cudaError_t attr_bf =
      cudaFuncSetAttribute(attn_pp_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPPSmem);
  if (f16 ? attr16 != cudaSuccess : attr_bf != cudaSuccess) return f16 ? attr16 : attr_bf;
  if (f16)
    attn_pp_kernel<true><<<a.ctas, kPPThreads, kPPSmem, s>>>(tq, tkv, a);
  else
    attn_pp_kernel<false><<<a.ctas, kPPThreads, kPPSmem, s>>>(tq, tkv, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || a.ctas < 2) return e;
  attn_pp_merge_kernel<<<dim3(a.ctas, 2), 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace vmla
