// gemm_bf16.cuh -- K14: float32-accurate products on the bf16 tensor cores, for the BitLinear
// backward (straight-through estimator).
//
//   D[i][j] = alpha * sum_k (Ahi[i][k] + Alo[i][k]) * B[j][k]
//
// A carries float32 values as bf16 pairs hi = bf16(a), lo = bf16(a - hi) (16 significant bits
// together, so a - hi - lo is within 2^-17 of |a|); B holds values bf16 represents exactly (the
// ternary codes, the int8 activation codes). A product of two bf16 values is exact in the float32
// accumulator, so D is the float32-accumulated product of a and B up to the rounding of lo and the
// order of the additions. Both operands are K-major in global memory ([rows][K], row pitch a
// multiple of 16 bytes). Per CTA: one 128 x 256 tile of D over a range of k-blocks; a producer
// thread stages 64-wide k-blocks of the hi and lo A tiles (128 rows) and the B tile (256 rows)
// with TMA (128-byte swizzle) into a 3-stage ring, one thread issues four tcgen05.mma.kind::f16
// (M 128, N 256, K 16) per operand pair and k-block into one float32 accumulator in tensor memory
// (256 columns), and the four warps read their 32 rows back (thread = row of D) and store 32
// consecutive columns at a time. With a K split (grid z) each CTA writes its raw partial tile to
// part[z], and bf16_gemm_reduce_kernel adds the partials in split order and applies alpha. Every
// wait is bounded; on a timeout the CTA drains its copies and MMAs and raises the device flag.
#pragma once

#include "common.cuh"

namespace mmf {
namespace gb {

constexpr int BM = 128;         // rows of D per CTA (MMA M)
constexpr int BN = 256;         // columns of D per CTA (MMA N)
constexpr int BK = 64;          // bf16 per k-block: one 128-byte swizzle atom
constexpr int UK = 16;          // K per kind::f16 instruction
constexpr int STAGES = 3;
constexpr int THREADS = 128;
constexpr int A_BYTES = BM * BK * 2;              // 16 KB
constexpr int B_BYTES = BN * BK * 2;              // 32 KB
constexpr int STAGE_BYTES = 2 * A_BYTES + B_BYTES;  // hi, lo, B
constexpr int NUM_BARS = 2 * STAGES + 2;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + NUM_BARS * 8 + 16;
constexpr uint32_t TMEM_COLS = BN;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct Params {
  CUtensorMap a_hi;     // [m][K] bf16, box 64 x 128, 128-byte swizzle
  CUtensorMap a_lo;     // same shape (unused when has_lo == 0)
  CUtensorMap b;        // [n][K] bf16, box 64 x 256, 128-byte swizzle
  int32_t m, n;         // D is m x n
  int32_t num_kb;       // k-blocks of K (the tail block reads zeros past K)
  int32_t kb_per_cta;   // k-blocks per split
  int32_t has_lo;
  const float* alpha;   // device scalar, or nullptr (1)
  float* d;             // [m][ldd], written when part == nullptr
  int64_t ldd;
  float* part;          // [gridDim.z][m][n] raw partials, or nullptr
  uint32_t wait_limit_us;
};

__global__ void __launch_bounds__(THREADS) bf16_gemm_kernel(const __grid_constant__ Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* full = bars;                   // TMA -> MMA          (count 1 + tx bytes)
  uint64_t* empty = bars + STAGES;         // MMA commit -> TMA   (count 1)
  uint64_t* accfull = bars + 2 * STAGES;   // MMA commit -> epilogue
  uint64_t* drain = accfull + 1;           // MMA drain after an abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int kb0 = blockIdx.z * P.kb_per_cta;
  const int kb1 = kb0 + P.kb_per_cta < P.num_kb ? kb0 + P.kb_per_cta : P.num_kb;
  const int nkb = kb1 - kb0;  // >= 1: the host sizes the split so that every CTA has work
  const uint32_t limit = P.wait_limit_us;
  const bool has_lo = P.has_lo != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&P.a_hi);
    if (has_lo) tma_prefetch_desc(&P.a_lo);
    tma_prefetch_desc(&P.b);
  }
  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int i = 0;
      for (; i < nkb; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_flag)) break;
        uint8_t* st = smem + s * STAGE_BYTES;
        const int kc = (kb0 + i) * BK;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(has_lo ? STAGE_BYTES : STAGE_BYTES - A_BYTES));
        tma_load_2d(st, &P.a_hi, kc, m0, &full[s]);
        if (has_lo) tma_load_2d(st + A_BYTES, &P.a_lo, kc, m0, &full[s]);
        tma_load_2d(st + 2 * A_BYTES, &P.b, kc, n0, &full[s]);
      }
      if (i < nkb) {
        // drain: the stages armed in the last STAGES iterations must see their copies land
        for (int j = i > STAGES ? i - STAGES : 0; j < i; ++j)
          mbar_wait_drain(&full[j % STAGES], (uint32_t)(j / STAGES) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // kind::f16: D float32 (bits 4-5 = 1), A and B bf16 (bits 7-9, 10-12 = 1), both K-major,
      // N >> 3 at bits 17-22, M >> 4 at bits 24-28
      constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                 ((uint32_t)(BM >> 4) << 24);
      int i = 0;
      for (; i < nkb; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!mbar_wait_bounded(&full[s], ph, limit, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
        const uint32_t b_addr = a_addr + 2 * A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / UK; ++kk) {
          const uint64_t bd = sw128_desc(b_addr + kk * UK * 2);
          tc_mma_bf16_ss(tmem, sw128_desc(a_addr + kk * UK * 2), bd, idesc, (i | kk) != 0 ? 1u : 0u);
          if (has_lo) tc_mma_bf16_ss(tmem, sw128_desc(a_addr + A_BYTES + kk * UK * 2), bd, idesc, 1u);
        }
        tc_commit(&empty[s]);
      }
      if (i == nkb) {
        tc_commit(accfull);
        // the accumulator is complete before this thread reaches the teardown barrier, whatever
        // happens to the epilogue's waits
        mbar_wait_drain(accfull, 0u);
      } else {
        tc_commit(drain);
        mbar_wait_drain(drain, 0u);
      }
    }
    __syncwarp();
  }

  // ------------------------------------------------------------------ epilogue (all four warps)
  bool have = mbar_wait_bounded(accfull, 0u, limit, abort_flag);
  have = __all_sync(0xffffffffu, have);
  if (have) {
    tc_fence_after();
    const int row = m0 + warp * 32 + lane;
    const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
    float* out = P.part ? P.part + ((int64_t)blockIdx.z * P.m + row) * P.n : P.d + (int64_t)row * P.ldd;
    const int64_t ld = P.part ? P.n : P.ldd;
    const float alpha = P.part || !P.alpha ? 1.0f : *P.alpha;
    const bool vec = ((reinterpret_cast<uintptr_t>(P.part ? P.part : P.d) | (uintptr_t)(ld * 4)) & 15u) == 0;
    for (int c0 = 0; c0 < BN && n0 + c0 < P.n; c0 += 32) {  // uniform across the CTA
      uint32_t v[32];
      tmem_ld_32x32b_x32(taddr + (uint32_t)c0, v);
      tmem_wait_ld();
      if (row < P.m) {
        float* o = out + n0 + c0;
        if (vec && n0 + c0 + 32 <= P.n) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(o + 4 * q) =
                make_float4(__uint_as_float(v[4 * q]) * alpha, __uint_as_float(v[4 * q + 1]) * alpha,
                            __uint_as_float(v[4 * q + 2]) * alpha, __uint_as_float(v[4 * q + 3]) * alpha);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (n0 + c0 + e < P.n) o[e] = __uint_as_float(v[e]) * alpha;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// d[i][j] = alpha * sum_z part[z][i][j] (alpha = 1 when alpha_p is null), the partials added in
// split order (deterministic); blockIdx.x = row i, 256 columns per block.
__global__ void __launch_bounds__(256) bf16_gemm_reduce_kernel(const float* __restrict__ part, int splits,
                                                               int32_t m, int32_t n, const float* alpha_p,
                                                               float* __restrict__ d, int64_t ldd) {
  const int64_t i = blockIdx.x;
  const int j = blockIdx.y * 256 + threadIdx.x;
  if (j >= n) return;
  const int64_t total = (int64_t)m * n;
  const float* p = part + i * n + j;
  float s = 0.0f;
  for (int z = 0; z < splits; ++z) s += p[(int64_t)z * total];
  d[i * ldd + j] = alpha_p ? s * *alpha_p : s;
}

}  // namespace gb
}  // namespace mmf
