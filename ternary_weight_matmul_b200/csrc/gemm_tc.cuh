// gemm_tc.cuh -- K2: ternary x int8 GEMM on the sm_100a tensor cores.
//
// Computes acc[row][n] = sum_k q[row][k] * t[n][k] exactly in int32 and applies the BitLinear
// epilogue. The product is laid out transposed on the MMA: the ternary weights are the A operand
// (M = 128 weight rows per tile) and the activation codes are the B operand (N = 128 tokens per
// tile), so the D accumulator is [weight row][token] in tensor memory.
//
//   * TMA stages the packed 2-bit weight tile (128 rows x 8 words = 4 KB) and the int8 activation
//     tile (128 tokens x 128 bytes, 128-byte swizzle = 16 KB) of every k-block into shared memory.
//   * Four expander warps turn the packed tile into int8 with byte permutes and write it straight
//     into tensor memory (tcgen05.st), one weight row per TMEM lane: no unpacked copy ever touches
//     shared memory, so the MMA reads only the activation tile from shared memory.
//   * One thread issues tcgen05.mma.kind::i8 (A from TMEM, B from shared memory, D in TMEM).
//   * Four epilogue warps read the int32 accumulators back with tcgen05.ld, rescale and store.
//   * The kernel is persistent (one CTA per SM) with a 6-stage operand ring and a double-buffered
//     accumulator, so the epilogue of one tile overlaps the MMAs of the next.
//
// Warp roles (320 threads): 0 = TMA producer, 1 = TMEM allocator + MMA issuer, 2..5 = expanders,
// 6..9 = epilogue. Every mbarrier wait is bounded; on a timeout the CTA drains its in-flight TMA
// copies and MMAs, releases its tensor memory and exits with the device timeout flag raised.
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace mmf {
namespace tc {

constexpr int BM = 128;      // weight rows per tile (MMA M)
constexpr int BN = 128;      // tokens per tile (MMA N)
constexpr int BK = 128;      // K per stage: one 128-byte swizzle atom of int8
constexpr int UK = 32;       // K per kind::i8 MMA instruction
constexpr int STAGES = 6;
constexpr int ACT_BYTES = BN * BK;       // 16 KB
constexpr int W_BYTES = BM * BK / 4;     // 4 KB (2 bits per code)
constexpr int W_WORDS_PER_ROW = BK / 16; // 8
constexpr int NUM_THREADS = 320;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;          // accumulators at columns [0, 128) and [128, 256)
constexpr uint32_t A_COL = 2 * BN;       // A stages at 256 + 32 * s (32 columns = 128 int8 per lane)
static_assert(A_COL + STAGES * (BK / 4) <= TMEM_COLS, "TMEM budget");

constexpr int SMEM_BAR_OFF = STAGES * (ACT_BYTES + W_BYTES);
constexpr int NUM_BARS = 3 * STAGES + 5;
constexpr int SMEM_BYTES = SMEM_BAR_OFF + NUM_BARS * 8 + 16 + 1024;  // + alignment slack

// Instruction descriptor, kind::i8: D = s32 (bits 4-5 = 2), A and B signed int8 (bits 7-9 and
// 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t IDESC = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

// Shared-memory matrix descriptor of a K-major, 128-byte-swizzled operand tile: start address
// >> 4 (bits 0-13), leading byte offset 16 B (unused for this layout, bits 16-29), stride byte
// offset 1024 B = 8 rows x 128 B (bits 32-45), descriptor version 1 (bits 46-47), layout type
// SWIZZLE_128B = 2 (bits 61-63).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  return (uint64_t)((smem_addr & 0x3FFFFu) >> 4) | ((uint64_t)1u << 16) | ((uint64_t)64u << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

struct Params {
  CUtensorMap act_map[3];  // int8 activation codes [m][ldq], box 128 x 128, swizzle 128B
  CUtensorMap w_map[3];    // u32 packed weights [n][kw], box 8 x 128
  GemmArgs g;
  int32_t m_tiles;
  int32_t tile_start[4];   // first tile of each segment; tile_start[nseg] = total
  int32_t num_kb;
  uint32_t wait_limit_us;
};

__device__ __forceinline__ void decode_tile(const Params& P, int tile, int& seg, int& nt, int& mt) {
  seg = 0;
  while (seg + 1 < P.g.nseg && tile >= P.tile_start[seg + 1]) ++seg;
  const int local = tile - P.tile_start[seg];
  nt = local / P.m_tiles;
  mt = local - nt * P.m_tiles;
}

// Wait without an abort check, used only while draining after an abort. Its own cap (1 s) does
// not follow the (possibly lowered) wait limit: copies and MMAs already issued complete within
// microseconds, and the CTA must not release shared or tensor memory before they have.
constexpr int64_t kDrainCycles = 1000000ll * kCyclesPerUs;
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const int64_t t0 = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t0 < kDrainCycles) {
  }
}

template <mmf_dtype YT>
__global__ void __launch_bounds__(NUM_THREADS, 1) ternary_gemm_tc_kernel(const __grid_constant__ Params P) {
  using OutT = typename Elem<YT>::T;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* act_s = smem;
  uint32_t* w_s = reinterpret_cast<uint32_t*>(smem + STAGES * ACT_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SMEM_BAR_OFF);
  uint64_t* full = bars;                   // TMA -> expanders      (count 1 + tx bytes)
  uint64_t* afull = bars + STAGES;         // expanders -> MMA      (count 4)
  uint64_t* empty = bars + 2 * STAGES;     // MMA commit -> producer (count 1)
  uint64_t* accfull = bars + 3 * STAGES;   // MMA commit -> epilogue (count 1), 2 buffers
  uint64_t* accempty = accfull + 2;        // epilogue -> MMA        (count 4), 2 buffers
  uint64_t* drain = accempty + 2;          // MMA drain after abort  (count 1)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = P.tile_start[P.g.nseg];
  const int num_kb = P.num_kb;
  const uint32_t limit = P.wait_limit_us;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], 4);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < P.g.nseg; ++s) {
      tma_prefetch_desc(&P.act_map[s]);
      tma_prefetch_desc(&P.w_map[s]);
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        int seg, nt, mt;
        decode_tile(P, tile, seg, nt, mt);
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], ACT_BYTES + W_BYTES);
          tma_load_2d(act_s + s * ACT_BYTES, &P.act_map[seg], kb * BK, mt * BN, &full[s]);
          tma_load_2d(w_s + s * (W_BYTES / 4), &P.w_map[seg], kb * W_WORDS_PER_ROW, nt * BM, &full[s]);
        }
      }
      if (!ok || *abort_flag) {
        // drain: every stage armed in the last STAGES iterations must see its copies land
        const uint32_t issued = it;
        for (uint32_t j = (issued > (uint32_t)STAGES ? issued - STAGES : 0); j < issued; ++j)
          mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tl = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++tl) {
        const uint32_t b = tl & 1u;
        if (!mbar_wait_bounded(&accempty[b], ((tl >> 1) & 1u) ^ 1u, limit, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ACC_COL + b * BN;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait_bounded(&afull[s], ph, limit, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_tmem = tmem_base + A_COL + s * (BK / 4);
          const uint32_t b_addr = smem_u32(act_s + s * ACT_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk)
            tc_mma_i8_ts(d_tmem, a_tmem + kk * (UK / 4), sw128_desc(b_addr + kk * UK), IDESC,
                         (kb | kk) != 0 ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&accfull[b]);
      }
      if (!ok || *abort_flag) {
        tc_commit(drain);
        mbar_wait_drain(drain, 0u);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------------ expanders
    const uint32_t sub = (uint32_t)(warp & 3);          // TMEM sub-partition of this warp
    const int row = (int)sub * 32 + lane;               // weight row within the tile = TMEM lane
    const uint32_t lane_addr = (sub * 32u) << 16;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        if (!mbar_wait_bounded(&full[s], ph, limit, abort_flag)) { ok = false; break; }
        const uint4* src = reinterpret_cast<const uint4*>(w_s + s * (W_BYTES / 4) + row * W_WORDS_PER_ROW);
        const uint4 p0 = src[0], p1 = src[1];
        uint32_t v[32];
        expand_word(p0.x, v + 0);
        expand_word(p0.y, v + 4);
        expand_word(p0.z, v + 8);
        expand_word(p0.w, v + 12);
        expand_word(p1.x, v + 16);
        expand_word(p1.y, v + 20);
        expand_word(p1.z, v + 24);
        expand_word(p1.w, v + 28);
        tmem_st_32x32b_x32(tmem_base + lane_addr + A_COL + s * (BK / 4), v);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[s]);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    // Thread = one weight row n (its TMEM lane); for each token column j of a 32-column chunk it
    // writes y[m0 + j][n]: the 32 lanes of a warp store 32 consecutive features of one token.
    // The per-token factor a/127 is loaded once per chunk (lane j holds token j) and broadcast.
    const uint32_t sub = (uint32_t)(warp & 3);
    const int row = (int)sub * 32 + lane;
    const uint32_t lane_addr = (sub * 32u) << 16;
    uint32_t tl = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tl) {
      const uint32_t b = tl & 1u;
      if (!mbar_wait_bounded(&accfull[b], (tl >> 1) & 1u, limit, abort_flag)) break;
      tc_fence_after();
      int seg, nt, mt;
      decode_tile(P, tile, seg, nt, mt);
      const GemmSeg* S = seg == 0 ? &P.g.seg[0] : (seg == 1 ? &P.g.seg[1] : &P.g.seg[2]);
      const int n = nt * BM + row;
      const bool nvalid = n < S->n;
      const float sw = S->sw[0];
      const float* deq = S->deq;
      OutT* y = reinterpret_cast<OutT*>(S->y);
      const int64_t ldy = S->ldy;
      const OutT* res = reinterpret_cast<const OutT*>(S->res);
      const int64_t ldres = S->ldres;
      int32_t* accp = S->acc;
      const int64_t ldacc = S->ldacc;
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + lane_addr + ACC_COL + b * BN + c0, v);
        tmem_wait_ld();
        const int64_t m0 = (int64_t)mt * BN + c0;
        const int64_t rem = P.g.m - m0;
        const int jmax = rem < 32 ? (int)rem : 32;
        const float dq = lane < jmax ? deq[m0 + lane] * sw : 0.0f;
        OutT* yp = y + m0 * ldy + S->ycol + n;
        const OutT* rp = res ? res + m0 * ldres + S->rescol + n : nullptr;
        int32_t* ap = accp ? accp + m0 * ldacc + n : nullptr;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float dj = __shfl_sync(0xffffffffu, dq, j);
          if (j < jmax && nvalid) {
            float z = (float)(int32_t)v[j] * dj;
            if (ap) ap[j * ldacc] = (int32_t)v[j];
            if (rp) z += Elem<YT>::load(rp + j * ldres);
            Elem<YT>::store(yp + j * ldy, z);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[b]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace tc
}  // namespace mmf
