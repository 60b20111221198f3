// tcgen05 GEMM kernels of the bf16 path (sm_100a).  All three are persistent
// (one CTA per SM taking work items in a grid-stride loop) and share one
// shape: A and B tiles staged in shared memory by TMA (128-byte swizzle) in a
// ring, one elected thread issuing tcgen05.mma into one of two TMEM
// accumulators, and four epilogue warps that read their TMEM lane (= output
// row) back with tcgen05.ld, park 64 rows at a time in shared memory and write
// them out contiguously, while the next item's loads and MMAs proceed.
//
//  * append_tc  [gist.it pt. 1, 3; paperlayer §3]: [c_KV | k_R] = W_down x,
//    rows placed in the ring slot of their frame (sink frames pinned, the
//    rest FIFO [paperlayer App. D.4]); k_R optionally rotated with the
//    absolute frame index.  K = d_model.
//  * qprep_tc   [paperlayer App. E, content-path absorption]: the query's
//    content part pushed through W_uk,h (q~ = W_uk,h^T q_nope, d_latent wide)
//    next to its rotated positional part.
//  * recon_tc   [gist.it pt. 2; paperlayer §3 On-demand reconstruction]: the
//    per-head dense entries k_h = [W_uk,h c | RoPE(k_R)], v_h = W_uv,h c.
#include <cuda_fp16.h>

#include "kernels.h"
#include "ptx.cuh"
#include "rope.cuh"

namespace vmla {
namespace {

constexpr int kThreads = 256;  // warp 0 TMA, warp 1 MMA (+TMEM alloc), warps 4..7 epilogue; every kernel is persistent

// Rotate NP adjacent pairs held in v[0..2 NP) at grid position (t, h, w).
template <int NP>
__device__ __forceinline__ void rotate_pairs(float (&v)[2 * NP], const Rope& rp, int t, int h, int w) {
#pragma unroll
  for (int p = 0; p < NP; ++p) rope_apply(v[2 * p], v[2 * p + 1], rope_cs(rp, p, t, h, w));
}
__device__ __forceinline__ void rotate16(float (&v)[32], const Rope& rp, int t, int h, int w) {
  rotate_pairs<16>(v, rp, t, h, w);
}

// (cos, sin) of every rotary pair at every position a chunk's queries take, one table per
// CTA: pair p of the t axis at chunk frame f sits at p * F + f, pair p of the h axis at row
// hh at n_t F + (p - n_t) grid_h + hh, pair p of the w axis at column ww after those.  Each
// entry is rope_cs of the same arguments, so a lookup equals the direct evaluation.
struct RopeTable {
  int F, gh, gw, n;  // chunk frames, grid rows, grid columns, entries
  __device__ __forceinline__ int index(const Rope& rp, int p, int f, int hh, int ww) const {
    return p < rp.n_t ? p * F + f
                      : (p < rp.n_t + rp.n_h ? rp.n_t * F + (p - rp.n_t) * gh + hh
                                             : rp.n_t * F + rp.n_h * gh + (p - rp.n_t - rp.n_h) * gw + ww);
  }
};
__device__ __forceinline__ RopeTable rope_table_shape(const Rope& rp, int n_q, const Ring& g) {
  RopeTable t;
  t.F = (n_q + g.tokens_per_frame - 1) / g.tokens_per_frame;
  t.gw = g.grid_w;
  t.gh = g.tokens_per_frame / g.grid_w;
  t.n = rp.n_t * t.F + rp.n_h * t.gh + rp.n_w * t.gw;
  return t;
}
// Fill the table (threads [tid0, tid0 + nthreads) of the caller take its entries in turn).
__device__ __forceinline__ void rope_table_fill(float2* tab, const RopeTable& t, const Rope& rp, int64_t t_first,
                                                int tid, int nthreads) {
  for (int e = tid; e < t.n; e += nthreads) {
    int p, pos;
    if (e < rp.n_t * t.F) {
      p = e / t.F;
      pos = (int)(t_first + e % t.F);
    } else if (e < rp.n_t * t.F + rp.n_h * t.gh) {
      const int k = e - rp.n_t * t.F;
      p = rp.n_t + k / t.gh;
      pos = k % t.gh;
    } else {
      const int k = e - rp.n_t * t.F - rp.n_h * t.gh;
      p = rp.n_t + rp.n_h + k / t.gw;
      pos = k % t.gw;
    }
    tab[e] = rope_cs(rp, p, pos, pos, pos);  // the pair's own axis picks pos
  }
}
template <int NP>
__device__ __forceinline__ void rotate_pairs_tab(float (&v)[2 * NP], const float2* tab, const RopeTable& t,
                                                 const Rope& rp, int f, int hh, int ww) {
#pragma unroll
  for (int p = 0; p < NP; ++p) rope_apply(v[2 * p], v[2 * p + 1], tab[t.index(rp, p, f, hh, ww)]);
}

// 32 floats as bf16 into 64 bytes of shared memory (16-byte aligned)
__device__ __forceinline__ void store_bf16x32_smem(uint8_t* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d[q] = make_uint4(pack_bf16x2(v[8 * q + 0], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                      pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
}

// N 16-byte chunks (8 bf16 each, from fp32 bit patterns in r) of row `row` of a column block
// parked for a TMA tensor store with 128-byte swizzle: the block holds 64 columns, 128 bytes per
// row, and chunk j of a row sits at position j ^ (row & 7), so the eight rows a quarter-warp
// writes at once fall in eight different bank groups.
// F16: the chunks are written as fp16 instead of bf16.
template <int N, bool F16 = false>
__device__ __forceinline__ void park_sw128(uint8_t* blk, int row, const uint32_t* r) {
  auto pk = [](float lo, float hi) { return F16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi); };
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const float* v = reinterpret_cast<const float*>(r + 8 * j);
    *reinterpret_cast<uint4*>(blk + row * 128 + ((j ^ (row & 7)) << 4)) =
        make_uint4(pk(v[0], v[1]), pk(v[2], v[3]), pk(v[4], v[5]), pk(v[6], v[7]));
  }
}

__device__ __forceinline__ void raw_to_float(const uint32_t (&r)[32], float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

// ============================================================== append
// Persistent: each CTA takes work items in a grid-stride loop.  An item is a
// column part of [c_KV | k_R] (NP pieces of N_PART columns) over MT consecutive
// 128-row tiles of the flattened (sample, row tile) sequence.  NP = 2 gives small
// calls -- one chunk of one sample, 37 row tiles -- work for twice as many SMs, at
// the price of reading x twice from L2.  MT = 2 reuses every W_down stage for two
// row tiles (two MMA chains, one accumulator each), which cuts the L2 -> SM bytes
// per row by a third when the row tiles outnumber the SMs.  With MT = 1 two TMEM
// accumulators alternate, so the epilogue of one item overlaps the loads and MMAs
// of the next; with MT = 2 the item's two accumulators fill TMEM and only the loads
// run ahead.  The epilogue parks the bf16 tile in shared memory, PARK rows at a
// time, and writes it out row-contiguous (ring rows of one frame are consecutive).
template <int N_PART, int MT = 1>
struct AppendCfg {
  static constexpr int A_BYTES = 128 * 128;  // 128 rows x 64 bf16
  static constexpr int B_BYTES = N_PART * 128;
  static constexpr int STAGE_BYTES = MT * A_BYTES + B_BYTES;
  static constexpr int OUT_STRIDE = N_PART * 2 + 16;  // bytes per parked row: an odd number of 16-byte chunks
  static constexpr int PARK = (212 * 1024 - 64 * OUT_STRIDE) / STAGE_BYTES >= 3 ? 64 : 32;  // rows parked at a time
  static constexpr int OUT_BYTES = PARK * OUT_STRIDE;
  static constexpr int FIT = (212 * 1024 - OUT_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = FIT > 8 ? 8 : FIT;
  static constexpr int NACC = 2 / MT;         // accumulator slots (items in flight between MMA and epilogue)
  static constexpr uint32_t TMEM_COLS = 512;  // 128-lane accumulators at columns 0 and 256
  static constexpr int SMEM_USED = 1024 + STAGES * STAGE_BYTES + OUT_BYTES + 2 * 128 * 8 + 256;
  // more than half of an SM's shared memory: one CTA per SM, so the 512 TMEM columns are always free
  static constexpr int SMEM = SMEM_USED > 116 * 1024 ? SMEM_USED : 116 * 1024;
  static_assert(N_PART % 16 == 0 && N_PART <= 256 && (MT == 1 || MT == 2), "bad N or MT");
  static_assert(B_BYTES % 1024 == 0 && OUT_BYTES % 16 == 0, "alignment");
  static_assert(STAGES >= 3 && SMEM <= 227 * 1024, "does not fit");
};

template <int N_PART, int MT>
__global__ void __launch_bounds__(kThreads, 1)
    append_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const AppendTc a, int n_parts, int tiles, int items) {
  using C = AppendCfg<N_PART, MT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sout = smem + C::STAGES * C::STAGE_BYTES;
  int64_t* row_lat = reinterpret_cast<int64_t*>(sout + C::OUT_BYTES);  // element offsets of each row's
  int64_t* row_pos = row_lat + 128;                                    // latent / positional destination
  uint64_t* full = reinterpret_cast<uint64_t*>(row_pos + 128);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_empty + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kblocks = a.d_model / 64;
  const int m_tiles = (a.rows + 127) / 128;
  const Guard g{abort_flag, a.err, a.limit_ns};

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * C::STAGES; ++i) mbar_init(&full[i], 1);  // full[], empty[]
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_full[1], 1);
    mbar_init(&acc_empty[0], 4);  // one arrival per epilogue warp
    mbar_init(&acc_empty[1], 4);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tslot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_w);
      int it = 0;  // global stage counter
      for (int item = blockIdx.x; item < items && !*abort_flag; item += gridDim.x) {
        const int part = item % n_parts, t0 = (item / n_parts) * MT, nt = min(MT, tiles - t0);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          if (!wait_phase(&empty[s], ((it / C::STAGES) & 1) ^ 1, g, DEV_ERR_TIMEOUT_PRODUCER)) break;
          uint8_t* sa = smem + s * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], nt * C::A_BYTES + C::B_BYTES);
          for (int u = 0; u < nt; ++u)
            tma_load_3d(sa + u * C::A_BYTES, &tm_x, &full[s], kb * 64, ((t0 + u) % m_tiles) * 128, (t0 + u) / m_tiles);
          tma_load_2d(sa + MT * C::A_BYTES, &tm_w, &full[s], kb * 64, part * N_PART);
        }
      }
      if (*abort_flag)  // let the copies in flight land before the CTA goes away
        for (int i = it > C::STAGES ? it - C::STAGES : 0; i < it; ++i)
          drain_phase(&full[i % C::STAGES], (i / C::STAGES) & 1, g);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, N_PART, false, false);
      int it = 0, j = 0;
      for (int item = blockIdx.x; item < items; item += gridDim.x, ++j) {
        const int acc = j % C::NACC, use = j / C::NACC;
        const int nt = min(MT, tiles - (item / n_parts) * MT);
        if (!wait_phase(&acc_empty[acc], (use & 1) ^ 1, g, DEV_ERR_TIMEOUT_MMA)) break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          if (!wait_phase(&full[s], (it / C::STAGES) & 1, g, DEV_ERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          const uint64_t bd = smem_desc(sa + MT * C::A_BYTES, 16, 1024, LAYOUT_SW128);
          for (int u = 0; u < nt; ++u) {  // one MMA chain per row tile, all on this W_down stage
            const uint32_t d = tbase + (acc * MT + u) * 256;
            const uint64_t ad = smem_desc(sa + u * C::A_BYTES, 16, 1024, LAYOUT_SW128);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              if (k == 0 && kb == 0)
                mma_ss_c<false>(d, desc_add(ad, k * 32), desc_add(bd, k * 32), idesc);
              else
                mma_ss_c<true>(d, desc_add(ad, k * 32), desc_add(bd, k * 32), idesc);
            }
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
      }
      mma_commit(done);
      if (*abort_flag) drain_phase(done, 0, g);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int wq = warp - 4, r = wq * 32 + lane, tid = threadIdx.x - 128;
    const int T = a.ring.tokens_per_frame;
    constexpr int CH = N_PART / 8;          // 16-byte chunks per row
    constexpr int WPP = C::PARK / 32;       // epilogue warps whose TMEM lanes fill one park
    int j = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x, ++j) {
      const int part = item % n_parts, t0 = (item / n_parts) * MT, nt = min(MT, tiles - t0);
      const int acc = j % C::NACC, use = j / C::NACC;
      const bool ok = wait_phase(&acc_full[acc], use & 1, g, DEV_ERR_TIMEOUT_EPILOGUE);
      __syncwarp();
      tc_fence_after();
#pragma unroll 1
      for (int u = 0; u < nt; ++u) {
        const int mt = (t0 + u) % m_tiles, b = (t0 + u) / m_tiles;
        const int m = mt * 128 + r;
        const int mm = m < a.rows ? m : 0;
        const int64_t frame = a.first_frame + mm / T;
        const int tok = mm % T;
        if (a.contiguous) {
          row_lat[r] = ((int64_t)b * a.rows + mm) * (a.d_latent + a.d_rope);
          row_pos[r] = row_lat[r] + a.d_latent;
        } else {
          const int64_t rr = (int64_t)b * a.ring_rows + ring_frame_slot(a.ring, frame) * T + tok;
          row_lat[r] = rr * a.d_latent;
          row_pos[r] = rr * a.d_rope;
        }
        named_bar_sync(1, 128);  // row table complete
        const int valid_rows = ok ? min(128, a.rows - mt * 128) : 0;
        const uint32_t col_base = (acc * MT + u) * 256;
#pragma unroll 1
        for (int pk = 0; pk < 128 / C::PARK; ++pk) {
          if (wq / WPP == pk) {  // warps of this park hold TMEM lanes PARK*pk .. PARK*pk + PARK - 1
            uint8_t* orow = sout + (r - C::PARK * pk) * C::OUT_STRIDE;
#pragma unroll 1
            for (int c0 = 0; c0 < N_PART; c0 += 16) {
              uint32_t raw[16];
              tmem_ld16(tmem_addr(tbase, wq * 32, col_base + c0), raw);
              float v[16];
#pragma unroll
              for (int q = 0; q < 16; ++q) v[q] = __uint_as_float(raw[q]);
              // 16 columns never straddle d_latent (a multiple of 64) nor d_latent + d_rope
              const int col = part * N_PART + c0;
              if (a.rotate && col >= a.d_latent && col < a.d_latent + a.d_rope) {
                const int p0 = (col - a.d_latent) >> 1;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                  rope_apply(v[2 * q], v[2 * q + 1],
                             rope_cs(a.rope, p0 + q, (int)frame, tok / a.ring.grid_w, tok % a.ring.grid_w));
              }
              uint4* o = reinterpret_cast<uint4*>(orow + c0 * 2);
              o[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                pack_bf16x2(v[6], v[7]));
              o[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                pack_bf16x2(v[14], v[15]));
            }
            tc_fence_before();
            __syncwarp();
            // after its last tile, each warp's lanes are read; all four free the slot for item j + NACC
            if (u == nt - 1 && lane == 0) mbar_arrive(&acc_empty[acc]);
          }
          named_bar_sync(1, 128);  // this park is complete
          const int rows_p = min(C::PARK, valid_rows - C::PARK * pk);
#pragma unroll 4
          for (int id = tid; id < rows_p * CH; id += 128) {
            const int row = id / CH, ch = id - row * CH;
            const int col = part * N_PART + ch * 8;
            if (col >= a.d_latent + a.d_rope) continue;  // the last part may run past [c_KV | k_R]
            const bool lat = col < a.d_latent;
            const int rt = C::PARK * pk + row;
            __nv_bfloat16* dst =
                (lat || a.contiguous ? a.ckv : a.kr) + (lat ? row_lat[rt] + col : row_pos[rt] + (col - a.d_latent));
            *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(sout + row * C::OUT_STRIDE + ch * 16);
          }
          named_bar_sync(1, 128);  // the park is written out before it is reused
        }
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

// ============================================================== q-absorb
// Persistent over (head, sample, 128-query tile) items: each CTA takes a contiguous
// run of them, so it meets one or two heads and keeps W_uk,h ([96 x 64] blocks, read
// as the MN-major B operand) resident, reloading it only when the head changes; the
// ring stages carry only the head's 128-column slice of q (two [128 x 64] blocks),
// which leaves room for a deeper prefetch.  Per item a single MMA chain of 6
// k-steps gives W_uk,h^T q_nope in TMEM (two accumulators alternate); two epilogue
// warpgroups park the item's rows of [q~_nope (d_c) | RoPE(q_rope) (32)] as 64-column
// blocks in the 128-byte swizzled layout (all 128 rows when they fit, else 64 at a
// time) -- the first the leading column blocks, the second the rest and the rotated
// positional part -- and TMA tensor stores write each park out, clipped at the last
// query; the stores run while the next item's positional part is rotated and its
// accumulator awaited.
template <int DL, int DR>
struct QPrepCfg {
  static constexpr int DN = 128 - DR;          // content dims of a head (the MMA's K)
  static constexpr int STAGE = 2 * 128 * 128;  // q[:, h*128 .. h*128+128) as two 64-col blocks
  static constexpr int WB = DN * 128;          // one 64-col block of W_uk,h: DN rows x 128 B
  static constexpr int W_BYTES = (DL / 64) * WB;
  static constexpr int ROW = DL + DR;                 // output row, elements
  static constexpr int NCB = (ROW + 63) / 64;        // 64-column blocks of a row (the last one partly used)
  static constexpr int PARK_ROWS = W_BYTES + 2 * STAGE + NCB * 128 * 128 <= 212 * 1024 ? 128 : 64;
  static constexpr int BLK = PARK_ROWS * 128;         // one parked column block
  static constexpr int OUT_BYTES = NCB * BLK;
  static constexpr int FIT = (212 * 1024 - OUT_BYTES - W_BYTES) / STAGE;
  static constexpr int STAGES = FIT > 4 ? 4 : FIT;
  static constexpr uint32_t TMEM_COLS = 512;          // two accumulators, at 0 and 256
  static constexpr int TAB_ENTRIES = 2048;            // (cos, sin) table of the chunk's positions
  static constexpr int SMEM_USED = 1024 + STAGES * STAGE + W_BYTES + OUT_BYTES + 256 + TAB_ENTRIES * 8;
  static constexpr int SMEM = SMEM_USED > 116 * 1024 ? SMEM_USED : 116 * 1024;  // one CTA per SM
  static constexpr int THREADS = 384;  // warp 0 TMA, warp 1 MMA, warps 4..11 two epilogue warpgroups
  static constexpr int NB = DL / 64;   // TMEM column blocks: [0, NA) parked by warpgroup 0,
  static constexpr int NA = (NB + 1) / 2;  // [NA, NB) and the positional block by warpgroup 1
  static_assert(DL % 64 == 0 && DL <= 256 && STAGES >= 2 && SMEM <= 227 * 1024, "bad d_latent");
  static_assert((DR == 16 || DR == 32 || DR == 64 || DR == 96) && W_BYTES % 1024 == 0, "rotary dims");
  static_assert(ROW > (NCB - 1) * 64 && ROW <= NCB * 64, "a row of q~ spans its parked column blocks");
};

template <int DL, int DR>
__global__ void __launch_bounds__(QPrepCfg<DL, DR>::THREADS, 1)
    qprep_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_wuk,
                    const __grid_constant__ CUtensorMap tm_out, const QPrepTc a, int items) {
  using C = QPrepCfg<DL, DR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sw = smem + C::STAGES * C::STAGE;  // the resident W_uk,h
  uint8_t* sout = sw + C::W_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sout + C::OUT_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_empty + 2;
  uint64_t* w_full = done + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(w_full + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);
  float2* rope_tab = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(full) + 256);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (a.n_q + 127) / 128;
  const int per_head = items / a.n_heads;  // (sample, query tile) items of one head
  const int beg = (int)((int64_t)blockIdx.x * items / gridDim.x);
  const int end = (int)((int64_t)(blockIdx.x + 1) * items / gridDim.x);
  const Guard g{abort_flag, a.err, a.limit_ns};

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * C::STAGES; ++i) mbar_init(&full[i], 1);  // full[], empty[]
    mbar_init(w_full, 1);
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_full[1], 1);
    mbar_init(&acc_empty[0], 8);  // one arrival per epilogue warp
    mbar_init(&acc_empty[1], 8);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tslot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_wuk);
      prefetch_tmap(&tm_out);
      int it = 0, cur_h = -1, wloads = 0;
      for (int item = beg; item < end && !*abort_flag; ++item, ++it) {
        const int h = item / per_head, mt = (item % per_head) % m_tiles, b = (item % per_head) / m_tiles;
        const int s = it % C::STAGES;
        if (h != cur_h) {
          // the MMAs of the previous item (the last readers of the old W_uk,h) have completed:
          // empty[] of its stage has finished the phase of that item's commit
          if (it > 0 && !wait_phase(&empty[(it - 1) % C::STAGES], ((it - 1) / C::STAGES) & 1, g,
                                    DEV_ERR_TIMEOUT_PRODUCER))
            break;
          mbar_arrive_expect_tx(w_full, C::W_BYTES);
          for (int cb = 0; cb < DL / 64; ++cb) tma_load_3d(sw + cb * C::WB, &tm_wuk, w_full, cb * 64, 0, h);
          cur_h = h;
          ++wloads;
        }
        if (!wait_phase(&empty[s], ((it / C::STAGES) & 1) ^ 1, g, DEV_ERR_TIMEOUT_PRODUCER)) break;
        uint8_t* st = smem + s * C::STAGE;
        mbar_arrive_expect_tx(&full[s], C::STAGE);
        tma_load_3d(st, &tm_q, &full[s], h * 128, mt * 128, b);
        tma_load_3d(st + 16384, &tm_q, &full[s], h * 128 + 64, mt * 128, b);
      }
      if (*abort_flag) {
        for (int i = it > C::STAGES ? it - C::STAGES : 0; i < it; ++i)
          drain_phase(&full[i % C::STAGES], (i / C::STAGES) & 1, g);
        if (wloads > 0) drain_phase(w_full, (wloads - 1) & 1, g);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, DL, false, true);
      const uint64_t bd = smem_desc(smem_u32(sw), C::WB, 1024, LAYOUT_SW128);
      int j = 0, cur_h = -1, wl = 0;
      for (int item = beg; item < end; ++item, ++j) {
        const int h = item / per_head;
        const int acc = j & 1, s = j % C::STAGES;
        if (!wait_phase(&acc_empty[acc], ((j >> 1) & 1) ^ 1, g, DEV_ERR_TIMEOUT_MMA)) break;
        if (h != cur_h) {
          if (!wait_phase(w_full, wl & 1, g, DEV_ERR_TIMEOUT_MMA)) break;
          cur_h = h;
          ++wl;
        }
        if (!wait_phase(&full[s], (j / C::STAGES) & 1, g, DEV_ERR_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * C::STAGE);
        const uint64_t ad = smem_desc(st, 16, 1024, LAYOUT_SW128);
#pragma unroll
        for (int kk = 0; kk < C::DN / 16; ++kk) {
          const uint64_t ak = desc_add(ad, (kk / 4) * 16384 + (kk % 4) * 32), bk = desc_add(bd, kk * 2048);
          if (kk == 0)
            mma_ss_c<false>(tbase + acc * 256, ak, bk, idesc);
          else
            mma_ss_c<true>(tbase + acc * 256, ak, bk, idesc);
        }
        mma_commit(&empty[s]);
        mma_commit(&acc_full[acc]);
      }
      mma_commit(done);
      if (*abort_flag) drain_phase(done, 0, g);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int wg = (warp - 4) >> 2, wq = warp & 3, r = wq * 32 + lane, tid = threadIdx.x - 128;
    const int T = a.ring.tokens_per_frame;
    const RopeTable tshape = rope_table_shape(a.rope, a.n_q, a.ring);
    const bool use_tab = tshape.n <= C::TAB_ENTRIES;
    if (use_tab) rope_table_fill(rope_tab, tshape, a.rope, a.t_first, tid, 256);
    named_bar_sync(1, 256);  // the table is complete
    // warpgroup 1 reads each item's positional part (DR * 2 bytes of its row) one item ahead
    constexpr int RQ = DR / 8;  // 16-byte pieces of it
    uint4 rq[RQ] = {};
    auto load_rope = [&](int item) {
      const int hh_ = item / per_head, mt_ = (item % per_head) % m_tiles, b_ = (item % per_head) / m_tiles;
      const int i_ = mt_ * 128 + r;
      const uint4* src = reinterpret_cast<const uint4*>(
          a.q + (((int64_t)b_ * a.n_q + (i_ < a.n_q ? i_ : 0)) * a.n_heads + hh_) * 128 + C::DN);
#pragma unroll
      for (int k = 0; k < RQ; ++k) rq[k] = src[k];
    };
    if (wg == 1 && beg < end) load_rope(beg);
    int j = 0;
    for (int item = beg; item < end; ++item, ++j) {
      const int h = item / per_head, mt = (item % per_head) % m_tiles, b = (item % per_head) / m_tiles;
      const int acc = j & 1;
      // the positional part does not wait for the tensor core
      float qr[DR];
      if (wg == 1) {
        const int i = mt * 128 + r;
        const int ii = i < a.n_q ? i : 0;
#pragma unroll
        for (int k = 0; k < RQ; ++k) {
          const uint32_t w4[4] = {rq[k].x, rq[k].y, rq[k].z, rq[k].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            qr[8 * k + 2 * e] = __uint_as_float(w4[e] << 16);
            qr[8 * k + 2 * e + 1] = __uint_as_float(w4[e] & 0xFFFF0000u);
          }
        }
        if (item + 1 < end) load_rope(item + 1);
        const int tok = ii % T;
        if (use_tab)
          rotate_pairs_tab<DR / 2>(qr, rope_tab, tshape, a.rope, ii / T, tok / a.ring.grid_w, tok % a.ring.grid_w);
        else
          rotate_pairs<DR / 2>(qr, a.rope, (int)(a.t_first + ii / T), tok / a.ring.grid_w, tok % a.ring.grid_w);
      }
      const bool ok = wait_phase(&acc_full[acc], (j >> 1) & 1, g, DEV_ERR_TIMEOUT_EPILOGUE);
      __syncwarp();
      tc_fence_after();
      const int valid_rows = ok ? min(128, a.n_q - mt * 128) : 0;
#pragma unroll 1
      for (int part = 0; part < 128 / C::PARK_ROWS; ++part) {
        if (tid == 0) bulk_wait_all_read();  // the previous park has been read by its stores
        named_bar_sync(1, 256);
        if ((r / C::PARK_ROWS) == part) {  // warps whose TMEM lanes are this park's rows
          const int pr = r - C::PARK_ROWS * part;
#pragma unroll 1
          for (int cb = wg ? C::NA : 0; cb < (wg ? C::NB : C::NA); ++cb) {
            uint32_t raw[64];
            tmem_ld64(tmem_addr(tbase, wq * 32, acc * 256 + cb * 64), raw);
            park_sw128<8>(sout + cb * C::BLK, pr, raw);
          }
          if (wg == 1) {  // the positional part: DR / 8 chunks from column block NB on, 8 per block
            constexpr int RC = DR / 8;
            park_sw128<(RC < 8 ? RC : 8)>(sout + C::NB * C::BLK, pr, reinterpret_cast<const uint32_t*>(qr));
            if constexpr (RC > 8)
              park_sw128<RC - 8>(sout + (C::NB + 1) * C::BLK, pr, reinterpret_cast<const uint32_t*>(qr) + 64);
          }
          fence_async_smem();  // the tensor stores (async proxy) read what these threads wrote
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[acc]);
        }
        named_bar_sync(1, 256);  // this park is complete
        if (tid == 0) {
          const int row0 = C::PARK_ROWS * part;
#pragma unroll 1
          for (int rb = 0; rb < C::PARK_ROWS; rb += 64) {
            if (row0 + rb >= valid_rows) break;
            for (int cb = 0; cb < C::NCB; ++cb)
              tma_store_3d(&tm_out, sout + cb * C::BLK + rb * 128, cb * 64, mt * 128 + row0 + rb, b * a.n_heads + h);
          }
          bulk_commit();
        }
      }
    }
    if (tid == 0) bulk_wait_all();  // the last stores have read shared memory and landed
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// ============================================================== per-head reconstruction
// Persistent over (sample, 128-row tile, head) items, head fastest, each CTA taking a
// contiguous run of them: the heads of a key tile follow each other in one CTA, which
// reads the tile's latents from L2 once per head and its positional keys once (one
// tile ahead), rotating them with the window-relative t when asked (reconstruct-once
// at read time) or the absolute frame (the dense cache).  Per item the
// reduction over d_latent runs through a ring of [128 rows x 64] latent blocks
// and [(d_nope + 128) x 64] blocks of [W_uk,h ; W_uv,h] (any d_latent a multiple of 64);
// two TMEM accumulators alternate so the epilogue of one item overlaps the
// next; two epilogue warpgroups park the item's 128 rows as [k_h (128) | v_h
// (128)] -- the first k_h (d_nope content columns from TMEM, then the d_rope
// positional columns), the second v_h.  With TMA_OUT (rows
// written to consecutive rows: the window of reconstruct-once) the park is four
// 128-byte-swizzled [128 x 64] blocks that four TMA tensor stores write out,
// clipped at the last key, while the threads go on to the next item; otherwise
// (rows to the ring slots of their frames: the dense cache) all 256 threads write
// each row's two 256-byte runs out contiguously.
__device__ __forceinline__ bool m_valid(int mt, int r, int rows) { return mt * 128 + r < rows; }

template <int DL, int DR, bool TMA_OUT = false>
struct ReconCfg {
  static constexpr int DN = 128 - DR;        // content dims of a head's key
  static constexpr int N = DN + 128;         // MMA N: [W_uk,h ; W_uv,h] rows
  static constexpr int NKB = DL / 64;
  static constexpr int A_BLK = 128 * 128;  // 128 latent rows x 64 cols
  static constexpr int B_BLK = N * 128;    // [d_nope rows of W_uk,h ; 128 rows of W_uv,h] x 64 cols
  static constexpr int STAGE = A_BLK + B_BLK;
  static constexpr int OUT_STRIDE = 256 * 2 + 16;  // parked row [k_h | v_h]: an odd number of 16-byte chunks
  static constexpr int OUT_BYTES = TMA_OUT ? 4 * 16384 : 128 * OUT_STRIDE;
  static constexpr int FIT = (212 * 1024 - OUT_BYTES) / STAGE;
  static constexpr int STAGES = FIT > 6 ? 6 : FIT;
  static constexpr uint32_t TMEM_COLS = 512;  // two accumulators of N columns, at 0 and 256
  static constexpr int TAB = 1024;  // (cos, sin) entries of the window's rotary positions (window_t)
  static constexpr int SMEM = 1024 + STAGES * STAGE + OUT_BYTES + 128 * 8 + 256 + TAB * 8;
  static constexpr int THREADS = 384;  // warp 0 TMA, warp 1 MMA, warps 4..11 two epilogue warpgroups
  static_assert(DR == 16 || DR == 32 || DR == 64 || DR == 96, "rotary dims");
  static_assert(N % 16 == 0 && N <= 256 && (DN * 128) % 1024 == 0, "MMA shape / swizzle atoms");
  static_assert(DL % 64 == 0 && STAGES >= 3 && SMEM <= 227 * 1024 && SMEM > 116 * 1024, "does not fit");
};

// 16 floats as bf16 (or fp16) into 32 bytes of shared memory (16-byte aligned); amax tracks the
// largest magnitude stored
template <bool F16>
__device__ __forceinline__ void store_x16_smem(uint8_t* dst, const float* v, float& amax) {
  uint4* d = reinterpret_cast<uint4*>(dst);
  auto pk = [](float lo, float hi) { return F16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi); };
#pragma unroll
  for (int q = 0; q < 2; ++q) {
#pragma unroll
    for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(v[8 * q + k]));
    d[q] = make_uint4(pk(v[8 * q + 0], v[8 * q + 1]), pk(v[8 * q + 2], v[8 * q + 3]), pk(v[8 * q + 4], v[8 * q + 5]),
                      pk(v[8 * q + 6], v[8 * q + 7]));
  }
}

// 16 floats as bf16 (or fp16) into columns c0 .. c0 + 15 (c0 a multiple of 16) of row r of a parked
// tile made of 128-byte-swizzled [128 x 64] blocks of 16 KB: 16-byte chunk j of a row's block at
// position j ^ (r & 7)
template <bool F16>
__device__ __forceinline__ void store_sw16_smem(uint8_t* tile, int r, int c0, const float* v, float& amax) {
  auto pk = [](float lo, float hi) { return F16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi); };
  uint8_t* row = tile + (c0 >> 6) * 16384 + r * 128;
  const int j = (c0 & 63) >> 3;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
#pragma unroll
    for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(v[8 * q + k]));
    *reinterpret_cast<uint4*>(row + (((j + q) ^ (r & 7)) << 4)) =
        make_uint4(pk(v[8 * q + 0], v[8 * q + 1]), pk(v[8 * q + 2], v[8 * q + 3]), pk(v[8 * q + 4], v[8 * q + 5]),
                   pk(v[8 * q + 6], v[8 * q + 7]));
  }
}

template <int DL, int DR, bool F16, bool TMA_OUT>
__global__ void __launch_bounds__(ReconCfg<DL, DR, TMA_OUT>::THREADS, 1)
    recon_tc_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_wuk,
                    const __grid_constant__ CUtensorMap tm_wuv, const __grid_constant__ CUtensorMap tm_out,
                    const ReconTc a, int items) {
  using C = ReconCfg<DL, DR, TMA_OUT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sout = smem + C::STAGES * C::STAGE;
  int64_t* row_k = reinterpret_cast<int64_t*>(sout + C::OUT_BYTES);  // element offset of each row's k_h
  uint64_t* full = reinterpret_cast<uint64_t*>(row_k + 128);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_empty + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);
  float2* rtab = reinterpret_cast<float2*>(sout + C::OUT_BYTES + 128 * 8 + 256);  // C::TAB entries
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (a.rows + 127) / 128;
  const Guard g{abort_flag, a.err, a.limit_ns};
  // window-relative rotation: (cos, sin) of every pair at every t of the window (0..W-1) and every
  // grid row and column, looked up per key (equal to the direct evaluation); wider windows or grids
  // than the table holds evaluate directly
  const RopeTable rt = rope_table_shape(a.rope, a.ring.window_frames * a.ring.tokens_per_frame, a.ring);
  const bool use_tab = a.window_t && !a.rotate && rt.n <= C::TAB;
  // a contiguous run of items per CTA (head fastest): the heads of a key tile follow each other,
  // so its positional keys are read and rotated once for all of them
  const int it_begin = (int)((int64_t)items * blockIdx.x / gridDim.x);
  const int it_end = (int)((int64_t)items * (blockIdx.x + 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * C::STAGES; ++i) mbar_init(&full[i], 1);  // full[], empty[]
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_full[1], 1);
    mbar_init(&acc_empty[0], 8);  // one arrival per epilogue warp
    mbar_init(&acc_empty[1], 8);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tslot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_c);
      prefetch_tmap(&tm_wuk);
      prefetch_tmap(&tm_wuv);
      int it = 0;
      for (int item = it_begin; item < it_end && !*abort_flag; ++item) {
        const int h = item % a.n_heads, mt = (item / a.n_heads) % m_tiles, b = item / (a.n_heads * m_tiles);
        for (int kb = 0; kb < C::NKB; ++kb, ++it) {
          const int s = it % C::STAGES;
          if (!wait_phase(&empty[s], ((it / C::STAGES) & 1) ^ 1, g, DEV_ERR_TIMEOUT_PRODUCER)) break;
          uint8_t* st = smem + s * C::STAGE;
          mbar_arrive_expect_tx(&full[s], C::STAGE);
          tma_load_3d(st, &tm_c, &full[s], kb * 64, mt * 128, b);
          tma_load_3d(st + C::A_BLK, &tm_wuk, &full[s], kb * 64, 0, h);
          tma_load_3d(st + C::A_BLK + C::DN * 128, &tm_wuv, &full[s], kb * 64, 0, h);
        }
      }
      if (*abort_flag)
        for (int i = it > C::STAGES ? it - C::STAGES : 0; i < it; ++i)
          drain_phase(&full[i % C::STAGES], (i / C::STAGES) & 1, g);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, C::N, false, false);
      int it = 0, j = 0;
      for (int item = it_begin; item < it_end; ++item, ++j) {
        const int acc = j & 1;
        if (!wait_phase(&acc_empty[acc], ((j >> 1) & 1) ^ 1, g, DEV_ERR_TIMEOUT_MMA)) break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < C::NKB; ++kb, ++it) {
          const int s = it % C::STAGES;
          if (!(ok = wait_phase(&full[s], (it / C::STAGES) & 1, g, DEV_ERR_TIMEOUT_MMA))) break;
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * C::STAGE);
          const uint64_t ad = smem_desc(st, 16, 1024, LAYOUT_SW128);
          const uint64_t bd = smem_desc(st + C::A_BLK, 16, 1024, LAYOUT_SW128);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (k == 0 && kb == 0)
              mma_ss_c<false>(tbase + acc * 256, desc_add(ad, k * 32), desc_add(bd, k * 32), idesc);
            else
              mma_ss_c<true>(tbase + acc * 256, desc_add(ad, k * 32), desc_add(bd, k * 32), idesc);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
      }
      mma_commit(done);
      if (*abort_flag) drain_phase(done, 0, g);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int wg = (warp - 4) >> 2, wq = warp & 3, r = wq * 32 + lane, tid = threadIdx.x - 128, wt = tid & 127;
    const int T = a.ring.tokens_per_frame;
    // warpgroup 0 reads each key tile's positional keys (DR * 2 bytes of its row) one tile ahead
    constexpr int RQ = DR / 8;  // 16-byte pieces of a positional key
    uint4 krq[RQ] = {};
    auto load_kr = [&](int item) {
      const int mt_ = (item / a.n_heads) % m_tiles, b_ = item / (a.n_heads * m_tiles);
      const int m_ = mt_ * 128 + r;
      if (m_ < a.rows) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.kr) +
                                                          ((int64_t)b_ * a.kr_rows + m_) * a.kr_stride);
#pragma unroll
        for (int k = 0; k < RQ; ++k) krq[k] = src[k];
      }
    };
    if (wg == 0 && it_begin < it_end) load_kr(it_begin);
    if (use_tab) rope_table_fill(rtab, rt, a.rope, 0, tid, 256);
    named_bar_sync(1, 256);  // the table is complete
    int j = 0;
    float kr[DR];      // warpgroup 0: this row's positional key, decoded and rotated, of key tile kr_tile
    int kr_tile = -1;
    for (int item = it_begin; item < it_end; ++item, ++j) {
      const int h = item % a.n_heads, mt = (item / a.n_heads) % m_tiles, b = item / (a.n_heads * m_tiles);
      const int acc = j & 1;
      if (wg == 0) {
        const int m = mt * 128 + r;
        const int mm = m < a.rows ? m : 0;
        const int64_t frame = a.first_frame + mm / T;
        const int tok = mm % T;
        const int64_t row = a.to_ring ? ring_frame_slot(a.ring, frame) * T + tok : mm;
        row_k[r] = (((int64_t)b * a.ring_rows + row) * 2 * a.n_heads + h) * 128;
        if (item / a.n_heads != kr_tile) {  // a new key tile: decode, prefetch the next, rotate
          kr_tile = item / a.n_heads;
#pragma unroll
          for (int k = 0; k < RQ; ++k) {
            const uint32_t w4[4] = {krq[k].x, krq[k].y, krq[k].z, krq[k].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {  // bf16 pairs
              kr[8 * k + 2 * e] = __uint_as_float(w4[e] << 16);
              kr[8 * k + 2 * e + 1] = __uint_as_float(w4[e] & 0xFFFF0000u);
            }
          }
          if ((kr_tile + 1) * a.n_heads < it_end) load_kr((kr_tile + 1) * a.n_heads);
          if (a.rotate || a.window_t) {
            // absolute frame, or the window-relative t of ring frame slot mm / T (to_ring 0)
            const int tt = a.rotate ? (int)frame : ring_slot_t(a.ring, mm / T, a.window_start_slot);
            if (use_tab)
              rotate_pairs_tab<DR / 2>(kr, rtab, rt, a.rope, tt, tok / a.ring.grid_w, tok % a.ring.grid_w);
            else
              rotate_pairs<DR / 2>(kr, a.rope, tt, tok / a.ring.grid_w, tok % a.ring.grid_w);
          }
        }
      }
      const bool ok = wait_phase(&acc_full[acc], (j >> 1) & 1, g, DEV_ERR_TIMEOUT_EPILOGUE);
      __syncwarp();
      tc_fence_after();
      const int valid_rows = ok ? min(128, a.rows - mt * 128) : 0;
      float amax = 0.f;
      // TMEM columns [c_begin, c_end) of this row (a multiple of 16 wide) through `put`, 32 per wait
      auto drain_cols = [&](int c_begin, int c_end, auto put) {
#pragma unroll 1
        for (int c0 = c_begin; c0 < c_end; c0 += 32) {
          if (c0 + 32 <= c_end) {
            uint32_t raw[32];
            tmem_ld32(tmem_addr(tbase, wq * 32, acc * 256 + c0), raw);
            put(c0 - c_begin, reinterpret_cast<const float*>(raw));
            put(c0 - c_begin + 16, reinterpret_cast<const float*>(raw) + 16);
          } else {
            uint32_t raw[16];
            tmem_ld16(tmem_addr(tbase, wq * 32, acc * 256 + c0), raw);
            put(c0 - c_begin, reinterpret_cast<const float*>(raw));
          }
        }
      };
      if constexpr (TMA_OUT) {
        // each warpgroup parks and stores its own half of the item (k_h: blocks 0 and 1, v_h: blocks
        // 2 and 3), waiting only for its own earlier stores and its own 128 threads
        uint8_t* park = sout + wg * 2 * 16384;
        if (wt == 0) bulk_wait_all_read();  // this warpgroup's previous stores have read its park
        named_bar_sync(2 + wg, 128);
        if (wg == 0) {  // k_h: TMEM columns 0..DN-1, then the positional part
          drain_cols(0, C::DN, [&](int c, const float* v) { store_sw16_smem<F16>(park, r, c, v, amax); });
#pragma unroll
          for (int c0 = 0; c0 < DR; c0 += 16) store_sw16_smem<F16>(park, r, C::DN + c0, kr + c0, amax);
        } else {  // v_h: TMEM columns DN..DN+127
          drain_cols(C::DN, C::DN + 128, [&](int c, const float* v) { store_sw16_smem<F16>(park, r, c, v, amax); });
        }
        fence_async_smem();  // the tensor stores (async proxy) read what these threads wrote
      } else {
        uint8_t* orow = sout + r * C::OUT_STRIDE;
        if (wg == 0) {  // TMEM columns 0..DN-1: the content part of k_h, then its positional part
          drain_cols(0, C::DN, [&](int c, const float* v) { store_x16_smem<F16>(orow + c * 2, v, amax); });
#pragma unroll
          for (int c0 = 0; c0 < DR; c0 += 16) store_x16_smem<F16>(orow + (C::DN + c0) * 2, kr + c0, amax);
        } else {  // TMEM columns DN..DN+127: v_h, parked from column 128
          drain_cols(C::DN, C::DN + 128,
                     [&](int c, const float* v) { store_x16_smem<F16>(orow + (128 + c) * 2, v, amax); });
        }
      }
      // fp16 holds magnitudes up to 65504: a row past it is reported, not stored as inf silently
      if (F16 && m_valid(mt, r, a.rows) && !(amax <= 65504.f)) atomicOr(a.err, DEV_ERR_RANGE);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);  // this warp's lanes are read
      if constexpr (TMA_OUT) {
        named_bar_sync(2 + wg, 128);  // this warpgroup's half of the item is parked
        if (wt == 0 && valid_rows > 0) {  // rows past the window are clipped by the tensor map
          for (int blk = 2 * wg; blk < 2 * wg + 2; ++blk)
            tma_store_3d(&tm_out, sout + blk * 16384, ((blk >> 1) * a.n_heads + h) * 128 + (blk & 1) * 64, mt * 128,
                         b);
          bulk_commit();
        }
      } else {
        named_bar_sync(1, 256);  // the item is parked and its row table complete
#pragma unroll 4
        for (int id = tid; id < valid_rows * 32; id += 256) {
          const int rr = id >> 5, ch = id & 31;
          uint16_t* dst = static_cast<uint16_t*>(a.dense) + row_k[rr] +
                          (ch < 16 ? ch * 8 : (int64_t)a.n_heads * 128 + (ch - 16) * 8);
          *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(sout + rr * C::OUT_STRIDE + ch * 16);
        }
        named_bar_sync(1, 256);  // the park is written out before it is reused
      }
    }
    if constexpr (TMA_OUT) {
      if (wt == 0) bulk_wait_all();  // this warpgroup's last stores have read shared memory and landed
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// ============================================================== folded output mixer
// out = O_bar W_fold^T, W_fold = [B_1 | ... | B_n_h], B_h = W_O,h W_uv,h [paperlayer App. E, value
// path absorbed into the output mixer]: one GEMM with K = n_h * d_c over the softmax-weighted
// latents of all heads.  O_bar arrives as a bf16 pair (rounded part + residual): two MMAs per
// k-step into one fp32 accumulator.  Persistent over (128-row tile, 128-column part) items,
// column part fastest so the CTAs working together share the O_bar rows in L2; K streamed in
// 64-column blocks through a 3-stage ring; two accumulators alternate; the epilogue parks the
// fp32 tile as four [128 x 32] SW128 boxes and stores them with TMA.
struct FoldCfg {
  static constexpr int BLK = 128 * 128;        // [128 rows x 64 bf16]
  static constexpr int STAGE = 3 * BLK;        // O_bar rounded, O_bar residual, W_fold rows
  static constexpr int STAGES = 3;
  static constexpr int OUT_BYTES = 4 * 16384;  // 128 rows x 128 fp32
  static constexpr uint32_t TMEM_COLS = 256;   // two accumulators of 128 columns
  static constexpr int SMEM = 1024 + STAGES * STAGE + OUT_BYTES + 256;
  static_assert(SMEM <= 227 * 1024, "does not fit");
};

__global__ void __launch_bounds__(kThreads, 1)
    fold_gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo,
                        const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_out,
                        const FoldTc a, int items) {
  using C = FoldCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sout = smem + C::STAGES * C::STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(sout + C::OUT_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_empty + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_parts = a.n_out / 128, kblocks = a.k / 64;
  const Guard g{abort_flag, a.err, a.limit_ns};

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * C::STAGES; ++i) mbar_init(&full[i], 1);  // full[], empty[]
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_full[1], 1);
    mbar_init(&acc_empty[0], 4);
    mbar_init(&acc_empty[1], 4);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tslot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_hi);
      prefetch_tmap(&tm_lo);
      prefetch_tmap(&tm_w);
      int it = 0;
      for (int item = blockIdx.x; item < items && !*abort_flag; item += gridDim.x) {
        const int np = item % n_parts, mt = item / n_parts;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          if (!wait_phase(&empty[s], ((it / C::STAGES) & 1) ^ 1, g, DEV_ERR_TIMEOUT_PRODUCER)) break;
          uint8_t* st = smem + s * C::STAGE;
          mbar_arrive_expect_tx(&full[s], C::STAGE);
          tma_load_3d(st, &tm_hi, &full[s], kb * 64, mt * 128, 0);
          tma_load_3d(st + C::BLK, &tm_lo, &full[s], kb * 64, mt * 128, 0);
          tma_load_3d(st + 2 * C::BLK, &tm_w, &full[s], kb * 64, np * 128, 0);
        }
      }
      if (*abort_flag)
        for (int i = it > C::STAGES ? it - C::STAGES : 0; i < it; ++i)
          drain_phase(&full[i % C::STAGES], (i / C::STAGES) & 1, g);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
      int it = 0, j = 0;
      for (int item = blockIdx.x; item < items; item += gridDim.x, ++j) {
        const int acc = j & 1;
        if (!wait_phase(&acc_empty[acc], ((j >> 1) & 1) ^ 1, g, DEV_ERR_TIMEOUT_MMA)) break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          if (!(ok = wait_phase(&full[s], (it / C::STAGES) & 1, g, DEV_ERR_TIMEOUT_MMA))) break;
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * C::STAGE);
          const uint64_t hd = smem_desc(st, 16, 1024, LAYOUT_SW128);
          const uint64_t ld = smem_desc(st + C::BLK, 16, 1024, LAYOUT_SW128);
          const uint64_t wd = smem_desc(st + 2 * C::BLK, 16, 1024, LAYOUT_SW128);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (k == 0 && kb == 0)
              mma_ss_c<false>(tbase + acc * 128, desc_add(hd, k * 32), desc_add(wd, k * 32), idesc);
            else
              mma_ss_c<true>(tbase + acc * 128, desc_add(hd, k * 32), desc_add(wd, k * 32), idesc);
            mma_ss_c<true>(tbase + acc * 128, desc_add(ld, k * 32), desc_add(wd, k * 32), idesc);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
      }
      mma_commit(done);
      if (*abort_flag) drain_phase(done, 0, g);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int wq = warp - 4, r = wq * 32 + lane, tid = threadIdx.x - 128;
    int j = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x, ++j) {
      const int np = item % n_parts, mt = item / n_parts;
      const int acc = j & 1;
      const bool ok = wait_phase(&acc_full[acc], (j >> 1) & 1, g, DEV_ERR_TIMEOUT_EPILOGUE);
      __syncwarp();
      tc_fence_after();
      if (tid == 0) bulk_wait_all_read();  // the previous tile's stores have read the parked image
      named_bar_sync(1, 128);
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem_addr(tbase, wq * 32, acc * 128 + c0), v);
        uint8_t* row = sout + (c0 >> 5) * 16384 + r * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4*>(row + ((q ^ (r & 7)) << 4)) = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      named_bar_sync(1, 128);
      if (tid == 0 && ok && !*abort_flag) {
        for (int blk = 0; blk < 4; ++blk) tma_store_3d(&tm_out, sout + blk * 16384, np * 128 + blk * 32, mt * 128, 0);
        bulk_commit();
      }
    }
    if (tid == 0) bulk_wait_all_read();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// B_h = W_O,h W_uv,h side by side (one-time weight preparation; fp32 sums, bf16 out):
// w_fold[o][h*d_c + c] = sum_e w_o[o][h*d_v + e] * w_uv[h][e][c]
__global__ void fold_weights_kernel(const __nv_bfloat16* w_o, const __nv_bfloat16* w_uv, __nv_bfloat16* w_fold,
                                    int d_out, int n_heads, int d_v, int d_c) {
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)d_out * n_heads * d_c;
  if (idx >= total) return;
  const int c = idx % d_c, h = (idx / d_c) % n_heads;
  const int64_t o = idx / ((int64_t)d_c * n_heads);
  const __nv_bfloat16* wo = w_o + o * n_heads * d_v + (int64_t)h * d_v;
  const __nv_bfloat16* wu = w_uv + (int64_t)h * d_v * d_c + c;
  float acc = 0.f;
  for (int e = 0; e < d_v; ++e) acc = fmaf(__bfloat162float(wo[e]), __bfloat162float(wu[(int64_t)e * d_c]), acc);
  w_fold[idx] = __float2bfloat16_rn(acc);
}

// ============================================================== query-latent absorption
// q~_h = [A_h c_Q | RoPE(W_qr,h c_Q)] with A_h = W_uk,h^T W_uq,h [paperlayer App. E content path,
// absorbed into the query latent c_Q; §4: d_q = 768]: per (sample, 128-query tile, head) item a
// GEMM over K = d_q with the stacked weights [A_h ; W_qr,h] ((d_c + 32) rows), streamed in
// 64-column blocks through a ring; the positional columns are rotated at the queries' positions
// in the epilogue, which parks the rows as 64-column blocks in the 128-byte swizzled layout and
// writes them with TMA tensor stores, clipped at the last query.
template <int DL, int DR>
struct QLatCfg {
  static constexpr int N = DL + DR;        // [A_h ; W_qr,h] rows: the MMA's N
  static constexpr int A_BLK = 128 * 128;
  static constexpr int B_BLK = N * 128;
  static constexpr int STAGE = A_BLK + B_BLK;
  static constexpr int NCB = (N + 63) / 64;  // 64-column blocks of a row (the last one partly used)
  static constexpr int BLK = 128 * 128;      // one parked column block of 128 rows
  static constexpr int OUT_BYTES = NCB * BLK;
  static constexpr int FIT = (212 * 1024 - OUT_BYTES) / STAGE;
  static constexpr int STAGES = FIT > 6 ? 6 : FIT;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int SMEM_USED = 1024 + STAGES * STAGE + OUT_BYTES + 256;
  static constexpr int SMEM = SMEM_USED > 116 * 1024 ? SMEM_USED : 116 * 1024;
  static_assert(DR % 16 == 0 && DR <= 96 && DL % 64 == 0, "rotary dims");
  static_assert(N % 16 == 0 && N <= 256 && B_BLK % 1024 == 0 && STAGES >= 2 && SMEM <= 227 * 1024, "bad d_latent");
};

template <int DL, int DR>
__global__ void __launch_bounds__(kThreads, 1)
    qlat_tc_kernel(const __grid_constant__ CUtensorMap tm_cq, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_out, const QLatTc a, int items) {
  using C = QLatCfg<DL, DR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sout = smem + C::STAGES * C::STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(sout + C::OUT_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_empty + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (a.n_q + 127) / 128, kblocks = a.d_q / 64;
  const Guard g{abort_flag, a.err, a.limit_ns};

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * C::STAGES; ++i) mbar_init(&full[i], 1);  // full[], empty[]
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_full[1], 1);
    mbar_init(&acc_empty[0], 4);
    mbar_init(&acc_empty[1], 4);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tslot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_cq);
      prefetch_tmap(&tm_w);
      prefetch_tmap(&tm_out);
      int it = 0;
      for (int item = blockIdx.x; item < items && !*abort_flag; item += gridDim.x) {
        const int h = item % a.n_heads, mt = (item / a.n_heads) % m_tiles, b = item / (a.n_heads * m_tiles);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          if (!wait_phase(&empty[s], ((it / C::STAGES) & 1) ^ 1, g, DEV_ERR_TIMEOUT_PRODUCER)) break;
          uint8_t* st = smem + s * C::STAGE;
          mbar_arrive_expect_tx(&full[s], C::STAGE);
          tma_load_3d(st, &tm_cq, &full[s], kb * 64, mt * 128, b);
          tma_load_3d(st + C::A_BLK, &tm_w, &full[s], kb * 64, 0, h);
        }
      }
      if (*abort_flag)
        for (int i = it > C::STAGES ? it - C::STAGES : 0; i < it; ++i)
          drain_phase(&full[i % C::STAGES], (i / C::STAGES) & 1, g);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, C::N, false, false);
      int it = 0, j = 0;
      for (int item = blockIdx.x; item < items; item += gridDim.x, ++j) {
        const int acc = j & 1;
        if (!wait_phase(&acc_empty[acc], ((j >> 1) & 1) ^ 1, g, DEV_ERR_TIMEOUT_MMA)) break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          if (!(ok = wait_phase(&full[s], (it / C::STAGES) & 1, g, DEV_ERR_TIMEOUT_MMA))) break;
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * C::STAGE);
          const uint64_t ad = smem_desc(st, 16, 1024, LAYOUT_SW128);
          const uint64_t bd = smem_desc(st + C::A_BLK, 16, 1024, LAYOUT_SW128);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (k == 0 && kb == 0)
              mma_ss_c<false>(tbase + acc * 256, desc_add(ad, k * 32), desc_add(bd, k * 32), idesc);
            else
              mma_ss_c<true>(tbase + acc * 256, desc_add(ad, k * 32), desc_add(bd, k * 32), idesc);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
      }
      mma_commit(done);
      if (*abort_flag) drain_phase(done, 0, g);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int wq = warp - 4, r = wq * 32 + lane, tid = threadIdx.x - 128;
    const int T = a.ring.tokens_per_frame;
    int j = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x, ++j) {
      const int h = item % a.n_heads, mt = (item / a.n_heads) % m_tiles, b = item / (a.n_heads * m_tiles);
      const int acc = j & 1;
      const int i = mt * 128 + r;
      const int ii = i < a.n_q ? i : 0;
      const int tok = ii % T;
      const int t = (int)(a.t_first + ii / T), hh = tok / a.ring.grid_w, ww = tok % a.ring.grid_w;
      const bool ok = wait_phase(&acc_full[acc], (j >> 1) & 1, g, DEV_ERR_TIMEOUT_EPILOGUE);
      __syncwarp();
      tc_fence_after();
      const int valid_rows = ok ? min(128, a.n_q - mt * 128) : 0;
      if (tid == 0) bulk_wait_all_read();  // the previous item's stores have read the parked rows
      named_bar_sync(1, 128);
#pragma unroll 1
      for (int cb = 0; cb < DL / 64; ++cb) {
        uint32_t raw[64];
        tmem_ld64(tmem_addr(tbase, wq * 32, acc * 256 + cb * 64), raw);
        park_sw128<8>(sout + cb * C::BLK, r, raw);
      }
      {
        float v[DR];  // the DR positional columns, rotated; parked 8 chunks of 8 per column block
#pragma unroll
        for (int c0 = 0; c0 < DR; c0 += 16) tmem_ld16(tmem_addr(tbase, wq * 32, acc * 256 + DL + c0),
                                                       *reinterpret_cast<uint32_t(*)[16]>(v + c0));
        rotate_pairs<DR / 2>(v, a.rope, t, hh, ww);
        constexpr int RC = DR / 8;
        park_sw128<(RC < 8 ? RC : 8)>(sout + (DL / 64) * C::BLK, r, reinterpret_cast<const uint32_t*>(v));
        if constexpr (RC > 8)
          park_sw128<RC - 8>(sout + (DL / 64 + 1) * C::BLK, r, reinterpret_cast<const uint32_t*>(v) + 64);
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      named_bar_sync(1, 128);
      if (tid == 0 && valid_rows > 0) {
#pragma unroll 1
        for (int rb = 0; rb < valid_rows; rb += 64)
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_store_3d(&tm_out, sout + cb * C::BLK + rb * 128, cb * 64, mt * 128 + rb, b * a.n_heads + h);
        bulk_commit();
      }
    }
    if (tid == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// [A_h ; W_qr,h] for every head (one-time weight preparation; fp32 sums, bf16 out):
// w_qabs[h][c][j] = sum_n w_uk[h][n][c] w_uq[h][n][j] (c < d_c), w_qr[h][c - d_c][j] (c >= d_c)
__global__ void fold_query_kernel(const __nv_bfloat16* w_uq, const __nv_bfloat16* w_qr, const __nv_bfloat16* w_uk,
                                  __nv_bfloat16* w_qabs, int n_heads, int d_nope, int d_rope, int d_c, int d_q) {
  const int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int rows = d_c + d_rope;
  if (idx >= (int64_t)n_heads * rows * d_q) return;
  const int jq = idx % d_q, c = (idx / d_q) % rows, h = idx / ((int64_t)d_q * rows);
  float acc = 0.f;
  if (c < d_c) {
    for (int n = 0; n < d_nope; ++n)
      acc = fmaf(__bfloat162float(w_uk[((int64_t)h * d_nope + n) * d_c + c]),
                 __bfloat162float(w_uq[((int64_t)h * d_nope + n) * d_q + jq]), acc);
  } else {
    acc = __bfloat162float(w_qr[((int64_t)h * d_rope + (c - d_c)) * d_q + jq]);
  }
  w_qabs[idx] = __float2bfloat16_rn(acc);
}

template <class K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int N_PART, int MT>
cudaError_t run_append(const CUtensorMap& tx, const CUtensorMap& tw, const AppendTc& a, int batch, int n_parts,
                       int ctas, cudaStream_t s) {
  using C = AppendCfg<N_PART, MT>;
  static const cudaError_t attr = set_smem(append_tc_kernel<N_PART, MT>, C::SMEM);
  if (attr != cudaSuccess) return attr;
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const int tiles = ((a.rows + 127) / 128) * batch;
  const int items = (tiles + MT - 1) / MT * n_parts;
  const int grid = std::min(items, ctas > 0 ? ctas : sms);
  append_tc_kernel<N_PART, MT><<<grid, kThreads, C::SMEM, s>>>(tx, tw, a, n_parts, tiles, items);
  return cudaGetLastError();
}

template <int N_OUT>
cudaError_t go_append(const CUtensorMap& tx, const CUtensorMap& tw, const AppendTc& a, int batch, cudaStream_t s,
                      const AppendPlan& p) {
  if constexpr (N_OUT <= 256) {
    if (p.parts == 1)
      return p.row_tiles == 2 ? run_append<N_OUT, 2>(tx, tw, a, batch, 1, p.ctas, s)
                              : run_append<N_OUT, 1>(tx, tw, a, batch, 1, p.ctas, s);
  }
  if constexpr (append_part_cols(N_OUT, 2) <= 256) {
    if (p.parts == 2) return run_append<append_part_cols(N_OUT, 2), 1>(tx, tw, a, batch, 2, p.ctas, s);
  }
  if (p.parts == 3) return run_append<append_part_cols(N_OUT, 3), 1>(tx, tw, a, batch, 3, p.ctas, s);
  return cudaErrorInvalidValue;
}

template <int DL, int DR>
cudaError_t go_qprep(const CUtensorMap& tq, const CUtensorMap& tw, const CUtensorMap& to, const QPrepTc& a, int batch,
                     cudaStream_t s) {
  using C = QPrepCfg<DL, DR>;
  static const cudaError_t attr = set_smem(qprep_tc_kernel<DL, DR>, C::SMEM);
  if (attr != cudaSuccess) return attr;
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const int items = ((a.n_q + 127) / 128) * a.n_heads * batch;
  qprep_tc_kernel<DL, DR><<<std::min(items, sms), C::THREADS, C::SMEM, s>>>(tq, tw, to, a, items);
  return cudaGetLastError();
}

template <int DR>
cudaError_t go_qprep_dl(const CUtensorMap& tq, const CUtensorMap& tw, const CUtensorMap& to, const QPrepTc& a,
                        int batch, cudaStream_t s) {
  switch (a.d_latent) {
    case 64: return go_qprep<64, DR>(tq, tw, to, a, batch, s);
    case 128: return go_qprep<128, DR>(tq, tw, to, a, batch, s);
    case 192: return go_qprep<192, DR>(tq, tw, to, a, batch, s);
    case 256:
      if constexpr (DR <= 32) return go_qprep<256, DR>(tq, tw, to, a, batch, s);
  }
  return cudaErrorInvalidValue;
}

// F16 runs are the reconstruct-once window (fp16 entries, consecutive rows: TMA tensor stores of the
// park through tm_out); the others the dense cache (bf16 entries placed in ring slots by the threads)
template <int DL, int DR, bool F16>
cudaError_t go_recon(const CUtensorMap& tc, const CUtensorMap& tuk, const CUtensorMap& tuv, const CUtensorMap& to,
                     const ReconTc& a, int batch, cudaStream_t s) {
  using C = ReconCfg<DL, DR, F16>;
  static const cudaError_t attr = set_smem(recon_tc_kernel<DL, DR, F16, F16>, C::SMEM);
  if (attr != cudaSuccess) return attr;
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const int items = ((a.rows + 127) / 128) * a.n_heads * batch;
  recon_tc_kernel<DL, DR, F16, F16><<<std::min(items, sms), C::THREADS, C::SMEM, s>>>(tc, tuk, tuv, to, a, items);
  return cudaGetLastError();
}

template <int DR, bool F16>
cudaError_t go_recon_dl(const CUtensorMap& tc, const CUtensorMap& tuk, const CUtensorMap& tuv, const CUtensorMap& to,
                        const ReconTc& a, int batch, cudaStream_t s) {
  switch (a.d_latent) {
    case 64: return go_recon<64, DR, F16>(tc, tuk, tuv, to, a, batch, s);
    case 128: return go_recon<128, DR, F16>(tc, tuk, tuv, to, a, batch, s);
    case 192: return go_recon<192, DR, F16>(tc, tuk, tuv, to, a, batch, s);
    case 256: return go_recon<256, DR, F16>(tc, tuk, tuv, to, a, batch, s);
    case 384:
      if constexpr (DR == 32) return go_recon<384, DR, F16>(tc, tuk, tuv, to, a, batch, s);
      break;
    case 512:
      if constexpr (DR == 32) return go_recon<512, DR, F16>(tc, tuk, tuv, to, a, batch, s);
      break;
  }
  return cudaErrorInvalidValue;
}

template <int DR>
cudaError_t go_recon_t(const CUtensorMap& tc, const CUtensorMap& tuk, const CUtensorMap& tuv, const CUtensorMap* to,
                       const ReconTc& a, int batch, cudaStream_t s) {
  if (a.f16) {
    if (!to || a.to_ring) return cudaErrorInvalidValue;
    return go_recon_dl<DR, true>(tc, tuk, tuv, *to, a, batch, s);
  }
  return go_recon_dl<DR, false>(tc, tuk, tuv, tc, a, batch, s);
}

}  // namespace


cudaError_t launch_fold_gemm_tc(const CUtensorMap& thi, const CUtensorMap& tlo, const CUtensorMap& tw,
                                const CUtensorMap& to, const FoldTc& a, cudaStream_t s) {
  if (a.rows <= 0) return cudaSuccess;
  if (a.k % 64 != 0 || a.n_out % 128 != 0) return cudaErrorInvalidValue;
  static const cudaError_t attr = set_smem(fold_gemm_tc_kernel, FoldCfg::SMEM);
  if (attr != cudaSuccess) return attr;
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const int items = ((a.rows + 127) / 128) * (a.n_out / 128);
  fold_gemm_tc_kernel<<<std::min(items, sms), kThreads, FoldCfg::SMEM, s>>>(thi, tlo, tw, to, a, items);
  return cudaGetLastError();
}

cudaError_t launch_fold_weights(const __nv_bfloat16* w_o, const __nv_bfloat16* w_uv, __nv_bfloat16* w_fold, int d_out,
                                int n_heads, int d_v, int d_c, cudaStream_t s) {
  const int64_t total = (int64_t)d_out * n_heads * d_c;
  if (total == 0) return cudaSuccess;
  fold_weights_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(w_o, w_uv, w_fold, d_out, n_heads, d_v, d_c);
  return cudaGetLastError();
}

template <int DL, int DR>
cudaError_t go_qlat(const CUtensorMap& tc, const CUtensorMap& tw, const CUtensorMap& to, const QLatTc& a, int batch,
                    cudaStream_t s) {
  if constexpr (DL + DR > 256) {
    return cudaErrorInvalidValue;
  } else {
    using C = QLatCfg<DL, DR>;
    static const cudaError_t attr = set_smem(qlat_tc_kernel<DL, DR>, C::SMEM);
    if (attr != cudaSuccess) return attr;
    static int sms = 0;
    if (sms == 0) {
      int dev = 0;
      cudaGetDevice(&dev);
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const int items = ((a.n_q + 127) / 128) * a.n_heads * batch;
    qlat_tc_kernel<DL, DR><<<std::min(items, sms), kThreads, C::SMEM, s>>>(tc, tw, to, a, items);
    return cudaGetLastError();
  }
}

template <int DR>
cudaError_t go_qlat_dl(const CUtensorMap& tc, const CUtensorMap& tw, const CUtensorMap& to, const QLatTc& a,
                       int batch, cudaStream_t s) {
  switch (a.d_latent) {
    case 64: return go_qlat<64, DR>(tc, tw, to, a, batch, s);
    case 128: return go_qlat<128, DR>(tc, tw, to, a, batch, s);
    case 192: return go_qlat<192, DR>(tc, tw, to, a, batch, s);
  }
  return cudaErrorInvalidValue;
}

bool qlat_supported(int d_latent, int d_rope, int d_q) {
  return (d_latent == 64 || d_latent == 128 || d_latent == 192) &&
         (d_rope == 16 || d_rope == 32 || d_rope == 64 || d_rope == 96) && d_latent + d_rope <= 256 && d_q > 0 &&
         d_q % 64 == 0;
}

cudaError_t launch_qlat_tc(const CUtensorMap& tc, const CUtensorMap& tw, const CUtensorMap& to, const QLatTc& a,
                           int batch, cudaStream_t s) {
  if (a.n_q <= 0) return cudaSuccess;
  if (!qlat_supported(a.d_latent, a.d_rope, a.d_q)) return cudaErrorInvalidValue;
  switch (a.d_rope) {
    case 16: return go_qlat_dl<16>(tc, tw, to, a, batch, s);
    case 32: return go_qlat_dl<32>(tc, tw, to, a, batch, s);
    case 64: return go_qlat_dl<64>(tc, tw, to, a, batch, s);
    case 96: return go_qlat_dl<96>(tc, tw, to, a, batch, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_fold_query(const __nv_bfloat16* w_uq, const __nv_bfloat16* w_qr, const __nv_bfloat16* w_uk,
                              __nv_bfloat16* w_qabs, int n_heads, int d_nope, int d_rope, int d_c, int d_q,
                              cudaStream_t s) {
  const int64_t total = (int64_t)n_heads * (d_c + d_rope) * d_q;
  if (total == 0) return cudaSuccess;
  fold_query_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(w_uq, w_qr, w_uk, w_qabs, n_heads, d_nope, d_rope,
                                                                   d_c, d_q);
  return cudaGetLastError();
}

AppendPlan append_tc_plan(int n_out, int rows, int batch, int n_split, int row_tiles, int ctas) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    cudaGetLastError();
  const int64_t tiles = (int64_t)((rows + 127) / 128) * batch;
  AppendPlan p{n_split, ctas, row_tiles};
  if (n_out > 512)
    p.parts = 3;
  else if (p.parts == 0)
    p.parts = (n_out > 256 || tiles < sms) ? 2 : 1;
  // two row tiles per item measured slower at every batch (Wan layer, batch 1 to 64: the item's two
  // accumulators fill TMEM, so its epilogue no longer overlaps the next item's MMAs)
  if (p.parts != 1 || p.row_tiles == 0) p.row_tiles = 1;
  return p;
}

cudaError_t launch_append_tc(const CUtensorMap& tx, const CUtensorMap& tw, const AppendTc& a, int batch,
                             cudaStream_t s, const AppendPlan& p) {
  if (a.rows <= 0) return cudaSuccess;
  if (a.d_model % 64 != 0) return cudaErrorInvalidValue;
  switch (a.d_latent + a.d_rope) {  // n_out = [c_KV | k_R] columns
    case 80: return go_append<80>(tx, tw, a, batch, s, p);    // d_rope 16
    case 144: return go_append<144>(tx, tw, a, batch, s, p);
    case 208: return go_append<208>(tx, tw, a, batch, s, p);
    case 272: return go_append<272>(tx, tw, a, batch, s, p);
    case 96: return go_append<96>(tx, tw, a, batch, s, p);    // d_rope 32
    case 160: return go_append<160>(tx, tw, a, batch, s, p);
    case 224: return go_append<224>(tx, tw, a, batch, s, p);
    case 288: return go_append<288>(tx, tw, a, batch, s, p);
    case 416: return go_append<416>(tx, tw, a, batch, s, p);
    case 544: return go_append<544>(tx, tw, a, batch, s, p);
    case 128: return go_append<128>(tx, tw, a, batch, s, p);  // d_rope 64
    case 192: return go_append<192>(tx, tw, a, batch, s, p);
    case 256: return go_append<256>(tx, tw, a, batch, s, p);
    case 320: return go_append<320>(tx, tw, a, batch, s, p);
    case 352: return go_append<352>(tx, tw, a, batch, s, p);  // d_rope 96 (160, 224, 288 above)
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_qprep_tc(const CUtensorMap& tq, const CUtensorMap& tw, const CUtensorMap& to, const QPrepTc& a,
                            int batch, cudaStream_t s) {
  if (a.n_q <= 0) return cudaSuccess;
  switch (a.d_rope) {
    case 16: return go_qprep_dl<16>(tq, tw, to, a, batch, s);
    case 32: return go_qprep_dl<32>(tq, tw, to, a, batch, s);
    case 64: return go_qprep_dl<64>(tq, tw, to, a, batch, s);
    case 96: return go_qprep_dl<96>(tq, tw, to, a, batch, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_recon_tc(const CUtensorMap& tc, const CUtensorMap& tuk, const CUtensorMap& tuv,
                            const CUtensorMap* to, const ReconTc& a, int batch, cudaStream_t s) {
  if (a.rows <= 0) return cudaSuccess;
  switch (a.d_rope) {
    case 16: return go_recon_t<16>(tc, tuk, tuv, to, a, batch, s);
    case 32: return go_recon_t<32>(tc, tuk, tuv, to, a, batch, s);
    case 64: return go_recon_t<64>(tc, tuk, tuv, to, a, batch, s);
    case 96: return go_recon_t<96>(tc, tuk, tuv, to, a, batch, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace vmla
