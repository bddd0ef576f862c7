// gemm_skinny.cuh -- ternary x int8 products of a few token rows (decode, B <= 64) on the sm_100a
// tensor cores, into exact int32 accumulators.
//
// acc[row][n] = sum_k q[row][k] * t[n][k] for row < m <= 64. The layout is the prefill GEMM's,
// transposed on the MMA (ternary weights = A operand, 128 weight rows per tile, expanded from their
// 2-bit fields into tensor memory; activation codes = B operand in shared memory, 128-byte swizzle),
// but the token dimension of a tile is only BN = 16, 32 or 64 columns, so an MMA does 8x to 2x less
// work than a 128-token tile, and the K dimension is split across the CTAs of a thread-block
// cluster so that a projection with few 128-row tiles still streams its weights on most SMs:
//   * one tile per CTA: weight rows n0 .. n0 + 127 of one segment, k-blocks [kb0, kb1) of 256;
//   * TMA brings each k-block's packed weights (8 KB) and codes (BN x 256 bytes, rows past m
//     zero-filled); four expander warps write the int8 weights into tensor memory; one thread
//     issues eight tcgen05.mma.kind::i8 (M 128, N BN, K 32) per k-block;
//   * four epilogue warps read the int32 accumulators back (one weight row per thread). With one
//     split they store them; otherwise every CTA of the cluster leaves its partial tile in its own
//     shared memory and, after a cluster barrier, CTA rank r sums rows [r * 128 / S, (r+1) * 128 / S)
//     of all S partials in rank order through distributed shared memory and stores them: an
//     exact, deterministic reduction with no atomics and nothing to clear beforehand.
// The epilogue of the projection (rescale, gates, residual, GLU) runs in the row stage that follows
// (decode_rows.cuh). Every mbarrier wait is bounded; an abandoned CTA still takes part in the
// cluster barriers (its partial counts as zero) and the timeout flag is raised.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace mmf {
namespace sk {

constexpr int BM = 128;
constexpr int BK = 256;
constexpr int UK = 32;
constexpr int STAGES = 4;
constexpr int W_WORDS_PER_ROW = BK / 16;  // 16 words = 64 bytes per weight row per stage
constexpr int W_BYTES = BM * BK / 4;      // 8 KB
constexpr int NUM_THREADS = 320;          // 0 TMA, 1 TMEM + MMA, 2..5 expanders, 6..9 epilogue
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t A_COL = 64;            // accumulator at columns [0, BN), A stages at 64 + 64 s
constexpr uint32_t A_COLS = BK / 4;
constexpr int MAX_SPLITS = 8;

template <int BN>
struct Layout {
  static constexpr int ACT_BOX_BYTES = BN * 128;        // BN rows x 128 bytes of K
  static constexpr int ACT_BYTES = 2 * ACT_BOX_BYTES;   // one 256-wide k-block
  static constexpr int W_OFF = STAGES * ACT_BYTES;
  static constexpr int RED_OFF = W_OFF + STAGES * W_BYTES;   // partial tile [BN][128] int32
  static constexpr int BAR_OFF = RED_OFF + BN * BM * 4;
  static constexpr int NUM_BARS = 4 * STAGES + 2;
  static constexpr int SMEM = BAR_OFF + NUM_BARS * 8 + 16 + 1024;
  // kind::i8: D s32, A and B signed int8, both K-major, N = BN, M = 128
  static constexpr uint32_t IDESC =
      (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
};

struct Params {
  CUtensorMap act_map[3];  // codes [m][ldq] int8, box 128 x BN, 128-byte swizzle
  CUtensorMap w_map[3];    // packed weights [n][kw] u32, box 16 x 128, 64-byte swizzle
  int32_t* acc[3];         // acc[seg][row * ldacc + n]
  int64_t ldacc;
  int32_t m;
  int32_t n[3];
  int32_t nseg;
  int32_t tile_start[4];   // first tile of each segment; tile_start[nseg] = total
  int32_t num_kb;
  int32_t splits;          // CTAs per tile (= cluster size), 1..8
  int32_t kb_per_split;
  uint32_t wait_limit_us;
};

template <int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1) ternary_gemm_skinny_kernel(const __grid_constant__ Params P) {
  using L = Layout<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* act_s = smem;
  uint32_t* w_s = reinterpret_cast<uint32_t*>(smem + L::W_OFF);
  int32_t* red_s = reinterpret_cast<int32_t*>(smem + L::RED_OFF);   // [token][row]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* full = bars;                 // TMA weights -> expanders (count 1 + tx bytes)
  uint64_t* afull = bars + STAGES;       // expanders -> MMA  (count 4)
  uint64_t* empty = bars + 2 * STAGES;   // MMA commit -> producer
  uint64_t* actfull = bars + 3 * STAGES; // TMA codes -> MMA (count 1 + tx bytes)
  uint64_t* accfull = bars + 4 * STAGES; // MMA commit -> epilogue
  uint64_t* drain = accfull + 1;         // MMA drain after an abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = P.splits;
  const int tile = blockIdx.x / S, split = blockIdx.x - tile * S;
  int seg = 0;
  while (seg + 1 < P.nseg && tile >= P.tile_start[seg + 1]) ++seg;
  const int n0 = (tile - P.tile_start[seg]) * BM;
  const int kb0 = split * P.kb_per_split;
  const int kb1 = min(P.num_kb, kb0 + P.kb_per_split);
  const int nkb = kb1 > kb0 ? kb1 - kb0 : 0;
  const uint32_t limit = P.wait_limit_us;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], 4);
      mbar_init(&empty[s], 1);
      mbar_init(&actfull[s], 1);
    }
    mbar_init(accfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&P.act_map[seg]);
    tma_prefetch_desc(&P.w_map[seg]);
  }
  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  uint32_t vals[BN];  // epilogue threads: the accumulators of their weight row
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // The weights do not depend on the preceding kernel: the first stages' weight tiles are
      // requested before waiting for it (programmatic dependent launch), the codes after.
      const int npro = nkb < STAGES ? nkb : STAGES;
      for (int it = 0; it < npro; ++it) {
        mbar_arrive_expect_tx(&full[it], W_BYTES);
        tma_load_2d(w_s + it * (W_BYTES / 4), &P.w_map[seg], (kb0 + it) * W_WORDS_PER_ROW, n0, &full[it]);
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int it = 0, wi = npro;  // stages whose codes / weights have been requested
      for (; it < nkb; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        if (it >= STAGES) {
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_flag)) break;
          mbar_arrive_expect_tx(&full[s], W_BYTES);
          tma_load_2d(w_s + s * (W_BYTES / 4), &P.w_map[seg], (kb0 + it) * W_WORDS_PER_ROW, n0, &full[s]);
          wi = it + 1;
        }
        const int kb = kb0 + it;
        mbar_arrive_expect_tx(&actfull[s], L::ACT_BYTES);
        uint8_t* ad = act_s + s * L::ACT_BYTES;
        tma_load_2d(ad, &P.act_map[seg], kb * BK, 0, &actfull[s]);
        tma_load_2d(ad + L::ACT_BOX_BYTES, &P.act_map[seg], kb * BK + 128, 0, &actfull[s]);
      }
      if (it < nkb) {
        // drain: every armed stage of the last STAGES iterations must see its copies land
        for (int j = wi > STAGES ? wi - STAGES : 0; j < wi; ++j)
          mbar_wait_drain(&full[j % STAGES], (uint32_t)(j / STAGES) & 1u);
        for (int j = it > STAGES ? it - STAGES : 0; j < it; ++j)
          mbar_wait_drain(&actfull[j % STAGES], (uint32_t)(j / STAGES) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0;
      for (; it < nkb; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        if (!mbar_wait_bounded(&afull[s], ph, limit, abort_flag)) break;
        if (!mbar_wait_bounded(&actfull[s], ph, limit, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_tmem = tmem_base + A_COL + s * A_COLS;
        const uint32_t b_addr = smem_u32(act_s + s * L::ACT_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / UK; ++kk)
          tc_mma_i8_ts(tmem_base, a_tmem + kk * (UK / 4),
                       sw128_desc(b_addr + (kk >> 2) * L::ACT_BOX_BYTES + (kk & 3) * UK), L::IDESC,
                       (it | kk) != 0 ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      if (it == nkb) {
        tc_commit(accfull);
        mbar_wait_drain(accfull, 0u);
      } else {
        tc_commit(drain);
        mbar_wait_drain(drain, 0u);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------------ expanders
    const uint32_t sub = (uint32_t)(warp & 3);
    const int row = (int)sub * 32 + lane;
    const uint32_t lane_addr = (sub * 32u) << 16;
    const uint32_t swz = (uint32_t)((row >> 1) & 3);  // the weight tile's 64-byte swizzle
    for (int it = 0; it < nkb; ++it) {
      const int s = it % STAGES;
      const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
      if (!mbar_wait_bounded(&full[s], ph, limit, abort_flag)) break;
      const uint4* src = reinterpret_cast<const uint4*>(w_s + s * (W_BYTES / 4) + row * W_WORDS_PER_ROW);
      const uint32_t ta = tmem_base + lane_addr + A_COL + s * A_COLS;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 p0 = src[(2 * h) ^ swz], p1 = src[(2 * h + 1) ^ swz];
        uint32_t v[32];
        expand_word(p0.x, v + 0);
        expand_word(p0.y, v + 4);
        expand_word(p0.z, v + 8);
        expand_word(p0.w, v + 12);
        expand_word(p1.x, v + 16);
        expand_word(p1.y, v + 20);
        expand_word(p1.z, v + 24);
        expand_word(p1.w, v + 28);
        tmem_st_32x32b_x32(ta + 32 * h, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[s]);
    }
  } else {
    // ------------------------------------------------------------------ epilogue: TMEM -> registers
    const uint32_t sub = (uint32_t)(warp & 3);
    const uint32_t lane_addr = (sub * 32u) << 16;
    bool got = nkb > 0 && mbar_wait_bounded(accfull, 0u, limit, abort_flag);
    got = __all_sync(0xffffffffu, got);
    if (got) {
      tc_fence_after();
      if (BN == 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem_base + lane_addr, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) vals[j] = v[j];
      } else {
#pragma unroll
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem_base + lane_addr + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) vals[c + j] = v[j];
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < BN; ++j) vals[j] = 0u;  // no k-blocks (or abandoned): contributes zero
    }
    const int row = (int)sub * 32 + lane;
    // the products are done: the next kernel (the row stage) may launch and wait for this one;
    // acc is still being read by the preceding kernel until it completes
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (S == 1) {
      const int n = n0 + row;
      if (n < P.n[seg]) {
#pragma unroll
        for (int j = 0; j < BN; ++j)
          if (j < P.m) P.acc[seg][(int64_t)j * P.ldacc + n] = (int32_t)vals[j];
      }
    } else {
#pragma unroll
      for (int j = 0; j < BN; ++j) red_s[j * BM + row] = (int32_t)vals[j];
    }
  }

  tc_fence_before();
  __syncthreads();
  if (S > 1) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();  // every CTA's partial tile is in its shared memory
    if (warp >= 6) {
      // rank `split` sums rows [r0, r0 + rows) of every partial, four rows per 16-byte load, all
      // of a thread's loads (up to 4 row quads x S ranks) in flight together
      const int rows = BM / S;
      const int r0 = split * rows;  // (cluster rank = split: the cluster spans one tile's splits)
      const int et = threadIdx.x - 6 * 32;
      const int rq = rows >> 2;     // row quads per token
      const int units = rq * P.m;
      const int4* peers[MAX_SPLITS];
#pragma unroll
      for (int p = 0; p < MAX_SPLITS; ++p)
        peers[p] = p < S ? reinterpret_cast<const int4*>(cluster.map_shared_rank(red_s, p)) : nullptr;
      for (int u0 = et; u0 < units; u0 += 4 * 128) {
        int4 acc4[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) acc4[t] = make_int4(0, 0, 0, 0);
#pragma unroll
        for (int p = 0; p < MAX_SPLITS; ++p) {
          if (p < S) {
            int4 v4[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const int u = u0 + t * 128;
              if (u < units) {
                const int j = u / rq, q = u - j * rq;
                v4[t] = peers[p][(j * BM + r0) / 4 + q];
              }
            }
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              acc4[t].x += v4[t].x; acc4[t].y += v4[t].y; acc4[t].z += v4[t].z; acc4[t].w += v4[t].w;
            }
          }
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int u = u0 + t * 128;
          if (u < units) {
            const int j = u / rq, q = u - j * rq;
            const int n = n0 + r0 + 4 * q;
            int32_t* dst = P.acc[seg] + (int64_t)j * P.ldacc + n;
            if (n + 3 < P.n[seg]) {
              *reinterpret_cast<int4*>(dst) = acc4[t];
            } else {
              const int32_t a4[4] = {acc4[t].x, acc4[t].y, acc4[t].z, acc4[t].w};
              for (int e = 0; e < 4; ++e)
                if (n + e < P.n[seg]) dst[e] = a4[e];
            }
          }
        }
      }
    }
    cluster.sync();  // peers have finished reading this CTA's partial tile
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace sk
}  // namespace mmf
