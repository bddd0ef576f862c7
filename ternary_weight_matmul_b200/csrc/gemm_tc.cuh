// gemm_tc.cuh -- K2: ternary x int8 GEMM on the sm_100a tensor cores.
//
// Computes acc[row][n] = sum_k q[row][k] * t[n][k] exactly in int32 and applies the BitLinear
// epilogue. The product is laid out transposed on the MMA: the ternary weights are the A operand
// (M = 128 weight rows per tile) and the activation codes are the B operand (N = 128 tokens per
// tile), so the D accumulator is [weight row][token] in tensor memory.
//
//   * TMA stages, per 256-wide k-block, the packed 2-bit weight tile (128 rows x 16 words = 8 KB,
//     64-byte swizzle) and the int8 activation tile (128 tokens x 256 bytes as two 128-byte-
//     swizzled boxes = 32 KB) into shared memory.
//   * Four expander warps turn the packed tile into int8 with byte permutes and write it straight
//     into tensor memory (tcgen05.st), one weight row per TMEM lane: no unpacked copy ever touches
//     shared memory, so the MMA reads only the activation tile from shared memory.
//   * One thread issues tcgen05.mma.kind::i8 (A from TMEM, B from shared memory, D in TMEM),
//     eight instructions per k-block between two barrier waits.
//   * Eight epilogue warps (two per TMEM sub-partition) read the int32 accumulators back with
//     tcgen05.ld, stage them transposed in shared memory, rescale, optionally add the residual or
//     form the SiLU-gated product of paired gate/up rows (GLU), and store whole row segments.
//   * The kernel is persistent (one CTA per SM) with a 4-stage operand ring and a double-buffered
//     accumulator, so the epilogue of one tile overlaps the MMAs of the next.
//
// Warp roles (448 threads): 0 = TMA producer, 1 = TMEM allocator + MMA issuer, 2..5 = expanders,
// 6..13 = epilogue. Every mbarrier wait is bounded; on a timeout the CTA drains its in-flight TMA
// copies and MMAs, releases its tensor memory and exits with the device timeout flag raised.
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace mmf {
namespace tc {

constexpr int BM = 128;      // weight rows per tile (MMA M)
constexpr int BN = 128;      // tokens per tile (MMA N)
constexpr int BK = 256;      // K per stage
constexpr int UK = 32;       // K per kind::i8 MMA instruction
constexpr int STAGES = 4;
constexpr int ACT_BOX = 128;                  // K bytes per activation box (one 128-byte swizzle atom)
constexpr int ACT_BOX_BYTES = BN * ACT_BOX;   // 16 KB
constexpr int ACT_BYTES = BN * BK;            // 32 KB per stage (two boxes)
constexpr int W_WORDS_PER_ROW = BK / 16;      // 16 words = 64 bytes per weight row per stage
constexpr int W_BYTES = BM * BK / 4;          // 8 KB (2 bits per code)
constexpr int GLU_ROWS = BM / 2;              // GLU tiles pair 64 gate rows with 64 up rows
constexpr int NUM_THREADS = 448;
constexpr int EPI_WARPS = 8;
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;          // accumulators at columns [0, 128) and [128, 256)
constexpr uint32_t A_COLS = BK / 4;      // TMEM columns of one expanded A stage (256 int8 per lane)
constexpr uint32_t A_COL = 2 * BN;       // A stages at 256 + 64 * s
static_assert(A_COL + STAGES * A_COLS <= TMEM_COLS, "TMEM budget");

// Epilogue staging: the raw int32 accumulators of a 64-token chunk, [64 tokens][128 rows], one
// 32 KB buffer (two chunks per tile; fewer, larger rounds measured faster than four 32-token
// rounds on two buffers). Within a token's 512-byte row the 16-byte chunk c sits at
// c ^ ((c >> 3) & 1), which keeps both the row-wise writes and the 32-byte piece reads free of
// bank conflicts.
constexpr int EPI_CHUNK = 64;
constexpr int EPI_BUF_BYTES = EPI_CHUNK * BM * 4;
constexpr int SMEM_W_OFF = STAGES * ACT_BYTES;
constexpr int SMEM_EPI_OFF = SMEM_W_OFF + STAGES * W_BYTES;
constexpr int SMEM_DQ_OFF = SMEM_EPI_OFF + EPI_BUF_BYTES;  // per-token (a/127)*s, 2 x BN floats
// residual tile (bf16 outputs), prefetched by the epilogue threads with cp.async before they wait
// for the tile's accumulators: [chunk][piece][8 values], each thread reading back what it copied
constexpr int RES_BYTES = BN * BM * 2;
constexpr int SMEM_RES_OFF = SMEM_DQ_OFF + 2 * BN * 4;
constexpr int SMEM_BAR_OFF = SMEM_RES_OFF + RES_BYTES;
constexpr int NUM_BARS = 3 * STAGES + 5;
constexpr int SMEM_BYTES = SMEM_BAR_OFF + NUM_BARS * 8 + 16 + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

__device__ __forceinline__ int epi_word(int r) {  // staged position of row r within a token row
  return r ^ (((r >> 5) & 1) << 2);
}

// Instruction descriptor, kind::i8: D = s32 (bits 4-5 = 2), A and B signed int8 (bits 7-9 and
// 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t IDESC = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

// float(a) for |a| < 2^22 without a conversion instruction: a + 1.5 * 2^23 laid into the
// mantissa of a float whose spacing is 1, minus that constant again (both steps exact).
__device__ __forceinline__ float acc_to_float(int32_t a) {
  return __fsub_rn(__int_as_float(a + 0x4B400000), 12582912.0f);
}

// z = float(a) * dj for eight accumulators (the branch is uniform across the launch).
__device__ __forceinline__ void scale8(const int32_t (&a)[8], float dj, bool small_acc, float (&z)[8]) {
  if (small_acc) {
#pragma unroll
    for (int e = 0; e < 8; ++e) z[e] = __fmul_rn(acc_to_float(a[e]), dj);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) z[e] = __fmul_rn((float)a[e], dj);
  }
}

struct Params {
  CUtensorMap act_map[3];  // int8 activation codes [m][ldq], box 128 x 128, swizzle 128B
  CUtensorMap w_map[3];    // u32 packed weights [n][kw], box 16 x 128 (GLU: 16 x 64), swizzle 64B
  GemmArgs g;
  int32_t m_tiles;
  int32_t tile_start[4];   // first tile of each segment; tile_start[nseg] = total
  int32_t num_kb;
  int32_t small_acc;       // every |acc| < 2^22 (127 * k), so acc_to_float is exact
  uint32_t wait_limit_us;
};

__device__ __forceinline__ void decode_tile(const Params& P, int tile, int& seg, int& nt, int& mt) {
  seg = 0;
  while (seg + 1 < P.g.nseg && tile >= P.tile_start[seg + 1]) ++seg;
  const int local = tile - P.tile_start[seg];
  nt = local / P.m_tiles;
  mt = local - nt * P.m_tiles;
}

// Whether the epilogue prefetches tile (segment S, weight tile nt)'s residual into shared memory:
// bf16 output, a residual, a full 128-row non-GLU tile, 16-byte aligned row segments.
template <mmf_dtype YT>
__device__ __forceinline__ bool res_prefetch(const GemmSeg* S, int nt) {
  if (YT != MMF_BF16 || !S->res || S->glu || S->n - nt * BM < BM) return false;
  const uintptr_t base = reinterpret_cast<uintptr_t>(S->res) + (uintptr_t)(S->rescol + nt * BM) * 2u;
  return ((base | (uintptr_t)(S->ldres * 2)) & 15u) == 0;
}

// OR of `pred` over the 256 epilogue threads (named barrier 1); every caller gets the result.
__device__ __forceinline__ bool epi_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0u;
}

// Eight values of one output row segment, bf16 or float32, 16- or 32-byte store.
template <mmf_dtype YT>
__device__ __forceinline__ void store8(typename Elem<YT>::T* p, const float (&z)[8]) {
  if (YT == MMF_F32) {
    float* f = reinterpret_cast<float*>(p);
    *reinterpret_cast<float4*>(f) = make_float4(z[0], z[1], z[2], z[3]);
    *reinterpret_cast<float4*>(f + 4) = make_float4(z[4], z[5], z[6], z[7]);
  } else {
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(z[2 * q], z[2 * q + 1]);
      o[q] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}
template <mmf_dtype YT>
__device__ __forceinline__ void add8(const typename Elem<YT>::T* p, float (&z)[8]) {
  if (YT == MMF_F32) {
    const float4 ra = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p));
    const float4 rb = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + 4);
    z[0] += ra.x; z[1] += ra.y; z[2] += ra.z; z[3] += ra.w;
    z[4] += rb.x; z[5] += rb.y; z[6] += rb.z; z[7] += rb.w;
  } else {
    const uint4 r = *reinterpret_cast<const uint4*>(p);
    const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 rf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rw[q]));
      z[2 * q] += rf.x;
      z[2 * q + 1] += rf.y;
    }
  }
}

template <mmf_dtype YT>
__global__ void __launch_bounds__(NUM_THREADS, 1) ternary_gemm_tc_kernel(const __grid_constant__ Params P) {
  using OutT = typename Elem<YT>::T;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* act_s = smem;
  uint32_t* w_s = reinterpret_cast<uint32_t*>(smem + SMEM_W_OFF);
  int32_t* epi_s = reinterpret_cast<int32_t*>(smem + SMEM_EPI_OFF);
  float* dq_s = reinterpret_cast<float*>(smem + SMEM_DQ_OFF);
  OutT* res_s = reinterpret_cast<OutT*>(smem + SMEM_RES_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SMEM_BAR_OFF);
  uint64_t* full = bars;                   // TMA -> expanders      (count 1 + tx bytes)
  uint64_t* afull = bars + STAGES;         // expanders -> MMA      (count 4)
  uint64_t* empty = bars + 2 * STAGES;     // MMA commit -> producer (count 1)
  uint64_t* accfull = bars + 3 * STAGES;   // MMA commit -> epilogue (count 1), 2 buffers
  uint64_t* accempty = accfull + 2;        // epilogue -> MMA        (count 8), 2 buffers
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
      mbar_init(&accempty[b], EPI_WARPS);
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
        const GemmSeg& S = P.g.seg[seg];
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], ACT_BYTES + W_BYTES);
          uint8_t* ad = act_s + s * ACT_BYTES;
          tma_load_2d(ad, &P.act_map[seg], kb * BK, mt * BN, &full[s]);
          tma_load_2d(ad + ACT_BOX_BYTES, &P.act_map[seg], kb * BK + ACT_BOX, mt * BN, &full[s]);
          uint32_t* wd = w_s + s * (W_BYTES / 4);
          if (S.glu) {
            // rows [0, 64) of the tile: gate rows 64 nt..; rows [64, 128): the paired up rows
            tma_load_2d(wd, &P.w_map[seg], kb * W_WORDS_PER_ROW, nt * GLU_ROWS, &full[s]);
            tma_load_2d(wd + GLU_ROWS * W_WORDS_PER_ROW, &P.w_map[seg], kb * W_WORDS_PER_ROW,
                        S.glu_inner + nt * GLU_ROWS, &full[s]);
          } else {
            tma_load_2d(wd, &P.w_map[seg], kb * W_WORDS_PER_ROW, nt * BM, &full[s]);
          }
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
          // afull implies the stage's TMA landed: the expanders waited on full[s] first
          if (!mbar_wait_bounded(&afull[s], ph, limit, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_tmem = tmem_base + A_COL + s * A_COLS;
          const uint32_t b_addr = smem_u32(act_s + s * ACT_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk)
            tc_mma_i8_ts(d_tmem, a_tmem + kk * (UK / 4),
                         sw128_desc(b_addr + (kk >> 2) * ACT_BOX_BYTES + (kk & 3) * UK), IDESC,
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
    // the weight tile arrives with the 64-byte swizzle: 16-byte chunk c of row r sits at
    // c ^ ((r >> 1) & 3), so the 32 rows a warp reads at once fall in distinct banks
    const uint32_t swz = (uint32_t)((row >> 1) & 3);
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        if (!mbar_wait_bounded(&full[s], ph, limit, abort_flag)) { ok = false; break; }
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
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    // Two phases per 64-token chunk. Phase 1: each warp loads its sub-partition's 32 weight rows
    // x 32 tokens (its half of the chunk, 16 at a time) of int32 accumulators from TMEM (thread =
    // row) and stores them to shared memory transposed, as [token][row] (one conflict-free 32-bit
    // store per element); the second chunk waits for the first one's reads of the single staging
    // buffer (a barrier). Phase 2: the 256 epilogue threads walk the chunk token-major in pieces of
    // 8 output columns, rescale by (a/127) * s of the token, add the residual (or, for a GLU
    // tile, form SiLU(gate) * up from rows r and 64 + r) and write 16- or 32-byte vectors, so
    // every global access covers whole row segments of the output.
    const uint32_t sub = (uint32_t)(warp & 3);
    const int half = (warp - 6) >> 2;        // which 32 tokens of a chunk this warp loads
    const int row = (int)sub * 32 + lane;
    const int srow = epi_word(row);
    const uint32_t lane_addr = (sub * 32u) << 16;
    const int etid = threadIdx.x - 6 * 32;  // 0..255
    const bool small_acc = P.small_acc != 0;
    uint32_t tl = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tl) {
      const uint32_t b = tl & 1u;
      int seg, nt, mt;
      decode_tile(P, tile, seg, nt, mt);
      {
        // bf16 residual of the whole tile into shared memory while the tile's MMAs may still
        // run: one cp.async group per chunk, each thread copying exactly the pieces it adds in
        // phase 2
        const GemmSeg* S = seg == 0 ? &P.g.seg[0] : (seg == 1 ? &P.g.seg[1] : &P.g.seg[2]);
        cp_async_wait<0>();  // (nothing in flight from the previous tile may land on the new copies)
        if (res_prefetch<YT>(S, nt)) {
          const OutT* rsrc = reinterpret_cast<const OutT*>(S->res) + S->rescol + nt * BM;
#pragma unroll
          for (int ci = 0; ci < BN / EPI_CHUNK; ++ci) {
#pragma unroll
            for (int itp = 0; itp < 4; ++itp) {
              const int pidx = etid + itp * EPI_THREADS;
              const int64_t m = (int64_t)mt * BN + ci * EPI_CHUNK + (pidx >> 4);
              if (m < P.g.m) cp_async16(res_s + (ci * 4 * EPI_THREADS + pidx) * 8, rsrc + m * S->ldres + (pidx & 15) * 8);
            }
            cp_async_commit();
          }
        }
      }
      const bool got = mbar_wait_bounded(&accfull[b], (tl >> 1) & 1u, limit, abort_flag);
      // The eight epilogue warps meet at named barrier 1 below, so they must agree on leaving:
      // if any of them gave up waiting, all of them leave (barrier reduction over 256 threads).
      if (epi_any(!got)) break;
      tc_fence_after();
      const GemmSeg* S = seg == 0 ? &P.g.seg[0] : (seg == 1 ? &P.g.seg[1] : &P.g.seg[2]);
      const bool glu = S->glu != 0;
      const int n0 = nt * (glu ? GLU_ROWS : BM);           // first output column of the tile
      const int nrows = glu ? GLU_ROWS : (S->n - n0 < BM ? S->n - n0 : BM);
      const float sw = S->sw[0];
      const float* deq = S->deq;
      OutT* y = reinterpret_cast<OutT*>(S->y) + S->ycol + n0;
      const int64_t ldy = S->ldy;
      const OutT* res = S->res ? reinterpret_cast<const OutT*>(S->res) + S->rescol + n0 : nullptr;
      const int64_t ldres = S->ldres;
      int32_t* accp = S->acc ? S->acc + n0 : nullptr;
      const int64_t ldacc = S->ldacc;
      const int32_t act = S->act;
      const int act_rows = S->act_cols - n0;  // rows of this tile (from 0) that take the activation
      // per-token factors of this tile, staged once (buffer by tile parity; published to all
      // epilogue threads by the named barrier of the first chunk)
      float* dq = dq_s + (tl & 1u) * BN;
      if (etid < BN) {
        const int64_t m = (int64_t)mt * BN + etid;
        dq[etid] = m < P.g.m ? deq[m] * sw : 0.0f;
      }
      // vectorised phase 2 needs every row segment 16-byte aligned and complete
      const bool vec_ok = nrows == (glu ? GLU_ROWS : BM) &&
          ((reinterpret_cast<uintptr_t>(y) | (uintptr_t)(ldy * sizeof(OutT))) & 15u) == 0 &&
          (!res || ((reinterpret_cast<uintptr_t>(res) | (uintptr_t)(ldres * sizeof(OutT))) & 15u) == 0) &&
          (!accp || ((reinterpret_cast<uintptr_t>(accp) | (uintptr_t)(ldacc * 4)) & 15u) == 0);
      const bool res_pf = res_prefetch<YT>(S, nt);  // the residual is in shared memory
      for (int c0 = 0; c0 < BN; c0 += EPI_CHUNK) {
        int32_t* buf = epi_s;
        if (c0 > 0) asm volatile("bar.sync 1, 256;" ::: "memory");  // the first round has read buf
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(tmem_base + lane_addr + ACC_COL + b * BN + c0 + 32 * half + 16 * hh, v);
          tmem_wait_ld();
          if (hh == 1 && c0 + EPI_CHUNK >= BN) {
            // the accumulator buffer is drained: hand it back to the MMA issuer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[b]);
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) buf[(32 * half + 16 * hh + j) * BM + srow] = (int32_t)v[j];
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        const int64_t m0 = (int64_t)mt * BN + c0;
        const int64_t rem = P.g.m - m0;
        const int jmax = rem < EPI_CHUNK ? (int)rem : EPI_CHUNK;
        if (vec_ok && glu) {
          // 64 tokens x 8 pieces of 8 output columns = 512 pieces, two per thread
#pragma unroll
          for (int itp = 0; itp < 2; ++itp) {
          const int pidx = etid + itp * EPI_THREADS;
          const int j = pidx >> 3, r8 = (pidx & 7) * 8;
          if (j < jmax) {
            const int32_t* bj = buf + j * BM;
            const int4 g0 = *reinterpret_cast<const int4*>(bj + epi_word(r8));
            const int4 g1 = *reinterpret_cast<const int4*>(bj + epi_word(r8 + 4));
            const int4 u0 = *reinterpret_cast<const int4*>(bj + epi_word(GLU_ROWS + r8));
            const int4 u1 = *reinterpret_cast<const int4*>(bj + epi_word(GLU_ROWS + r8 + 4));
            const int32_t ga[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            const int32_t ua[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            const float dj = dq[c0 + j];
            float gv[8], z[8];
            scale8(ga, dj, small_acc, gv);
            scale8(ua, dj, small_acc, z);
#pragma unroll
            for (int e = 0; e < 8; ++e) z[e] = siluf_(gv[e]) * z[e];
            store8<YT>(y + (m0 + j) * ldy + r8, z);
          }
          }
        } else if (vec_ok) {
          // 64 tokens x 16 pieces of 8 rows = 1024 pieces, 4 per thread; a warp writes two whole
          // 128-row segments at a time (256 B in bf16, 512 B in fp32)
#pragma unroll
          for (int itp = 0; itp < 4; ++itp) {
            const int pidx = etid + itp * EPI_THREADS;
            const int j = pidx >> 4, r8 = (pidx & 15) * 8;
            if (j < jmax) {
              const int64_t m = m0 + j;
              const int32_t* bj = buf + j * BM;
              const int4 a0 = *reinterpret_cast<const int4*>(bj + epi_word(r8));
              const int4 a1 = *reinterpret_cast<const int4*>(bj + epi_word(r8 + 4));
              const int32_t aa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
              const float dj = dq[c0 + j];
              float z[8];
              scale8(aa, dj, small_acc, z);
              if (accp) {
                *reinterpret_cast<int4*>(accp + m * ldacc + r8) = a0;
                *reinterpret_cast<int4*>(accp + m * ldacc + r8 + 4) = a1;
              }
              if (res_pf) {
                // this chunk's cp.async group (and the earlier ones) have landed
                const int ci = c0 / EPI_CHUNK;
                if (ci == 0) cp_async_wait<1>();
                else cp_async_wait<0>();
                add8<YT>(res_s + (ci * 4 * EPI_THREADS + pidx) * 8, z);
              } else if (res) {
                add8<YT>(res + m * ldres + r8, z);
              }
              if (act != kActNone) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  if (r8 + e < act_rows) z[e] = apply_act(act, z[e]);
              }
              store8<YT>(y + m * ldy + r8, z);
            }
          }
        } else if (glu) {
          // unaligned GLU output: one output column per step
          for (int e = etid; e < EPI_CHUNK * GLU_ROWS; e += EPI_THREADS) {
            const int j = e / GLU_ROWS, r = e - j * GLU_ROWS;
            if (j >= jmax) break;
            const float dj = dq[c0 + j];
            const float gv = __fmul_rn((float)buf[j * BM + epi_word(r)], dj);
            const float uv = __fmul_rn((float)buf[j * BM + epi_word(GLU_ROWS + r)], dj);
            Elem<YT>::store(y + (m0 + j) * ldy + r, siluf_(gv) * uv);
          }
        } else {
          // ragged tile or unaligned output: one element per step, still token-major
          for (int e = etid; e < EPI_CHUNK * BM; e += EPI_THREADS) {
            const int j = e / BM, r = e - j * BM;
            if (j >= jmax) break;
            if (r >= nrows) continue;
            const int64_t m = m0 + j;
            const int32_t a = buf[j * BM + epi_word(r)];
            float z = __fmul_rn((float)a, dq[c0 + j]);
            if (accp) accp[m * ldacc + r] = a;
            if (res) z += Elem<YT>::load(res + m * ldres + r);
            if (r < act_rows) z = apply_act(act, z);
            Elem<YT>::store(y + m * ldy + r, z);
          }
        }
      }
    }
  }

  cp_async_wait<0>();  // epilogue threads: residual copies of an abandoned tile
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace tc
}  // namespace mmf
