// head.cuh -- K10: tied language-model head and greedy next token (generation).
//
// logits = RMSNorm(x) . E^T with E the embedding table [vocab][d] that the input embedding
// shares, then next = argmax (lowest index among equal maxima). Only the last position of each
// sequence is needed to generate, so this runs on a handful of token rows and streams the table
// once per pass: an HBM-bound product. Two forms:
//   * CUDA cores (any table dtype, up to kRows token rows a pass): every CTA normalises the rows
//     into shared memory in float32; each warp forms the logits of its vocabulary rows from
//     16-byte table loads with float32 accumulation and keeps a running (maximum, lowest index)
//     per token row.
//   * Tensor cores (bf16 table, up to kTcRowsMax token rows a pass): a small kernel writes the
//     normalised rows as bf16 hi / lo pairs, then tcgen05.mma.kind::f16 forms 128 vocabulary rows
//     of logits per CTA from TMA-staged table tiles (below).
// Either way the CTA's best per token row goes to a partial array that a one-warp-per-row kernel
// reduces to the ids.
#pragma once

#include "common.cuh"

namespace mmf {
namespace head {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 8;          // token rows per pass (the host loops over groups of 8)
constexpr int kMinRowsPerCta = 16;

struct Args {
  const void* x;        // [b][d] (row group: b <= kRows rows starting here)
  mmf_dtype xdt;
  int32_t b;
  int32_t d;            // multiple of 8
  const float* norm_w;  // [d], nullable (= 1)
  float eps;
  const void* table;    // [vocab][d]
  mmf_dtype tdt;
  int32_t vocab;
  int32_t rows_per_cta; // vocabulary rows per CTA
  float* logits;        // nullable [b][ld_logits]
  int64_t ld_logits;
  float* pmax;          // [gridDim][kRows] best logit per (CTA, token row)
  int32_t* pidx;        // [gridDim][kRows] its vocabulary index
};

template <mmf_dtype DT>
__device__ __forceinline__ void row8(const void* base, int64_t idx, float (&o)[8]) {
  if (DT == MMF_F32) {
    const float4 p = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx));
    const float4 q = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx + 4));
    o[0] = p.x; o[1] = p.y; o[2] = p.z; o[3] = p.w; o[4] = q.x; o[5] = q.y; o[6] = q.z; o[7] = q.w;
  } else {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(base) + idx));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      o[2 * q] = __uint_as_float(w[q] << 16);
      o[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
    }
  }
}

// Eight table values as raw words (one 16-byte word for bf16, two for float32), loaded one chunk
// ahead of their use.
template <mmf_dtype DT> struct Raw8h { uint4 w[DT == MMF_F32 ? 2 : 1]; };
template <mmf_dtype DT>
__device__ __forceinline__ void raw8h_load(const void* base, int64_t idx, Raw8h<DT>& r) {
  if (DT == MMF_F32) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(base) + idx);
    r.w[0] = __ldcs(p);
    r.w[DT == MMF_F32 ? 1 : 0] = __ldcs(p + 1);
  } else {
    r.w[0] = __ldcs(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(base) + idx));
  }
}
template <mmf_dtype DT>
__device__ __forceinline__ void raw8h_unpack(const Raw8h<DT>& r, float (&o)[8]) {
  if (DT == MMF_F32) {
    const uint4 a = r.w[0], b = r.w[DT == MMF_F32 ? 1 : 0];
    o[0] = __uint_as_float(a.x); o[1] = __uint_as_float(a.y); o[2] = __uint_as_float(a.z); o[3] = __uint_as_float(a.w);
    o[4] = __uint_as_float(b.x); o[5] = __uint_as_float(b.y); o[6] = __uint_as_float(b.z); o[7] = __uint_as_float(b.w);
  } else {
    const uint32_t w[4] = {r.w[0].x, r.w[0].y, r.w[0].z, r.w[0].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      o[2 * q] = __uint_as_float(w[q] << 16);
      o[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
    }
  }
}

// Better of two (logit, index) candidates: the larger logit, the lower index on equal logits.
__device__ __forceinline__ bool head_better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

template <mmf_dtype XT, mmf_dtype TT, int NB>
__global__ void __launch_bounds__(kThreads, 2) head_logits_kernel(const Args a) {
  extern __shared__ __align__(16) float rs[];   // [NB][2][d/2]: normalised rows, halves of chunks
  __shared__ float red[kWarps][kRows];
  __shared__ float wbest[kWarps][kRows];
  __shared__ int wbidx[kWarps][kRows];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = a.d, nck = d >> 3;
  // 1. r = x / rms(x) * w for every token row, float32 (every CTA the same)
  float ss[NB];
#pragma unroll
  for (int r = 0; r < NB; ++r) ss[r] = 0.0f;
  for (int c = threadIdx.x; c < nck; c += kThreads) {
#pragma unroll
    for (int r = 0; r < NB; ++r) {
      float v[8];
      row8<XT>(a.x, (int64_t)r * d + 8 * c, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss[r] = fmaf(v[e], v[e], ss[r]);
    }
  }
#pragma unroll
  for (int r = 0; r < NB; ++r) {
    const float t = warp_sum(ss[r]);
    if (lane == 0) red[warp][r] = t;
  }
  __syncthreads();
  float rinv[NB];
#pragma unroll
  for (int r = 0; r < NB; ++r) {
    float t = 0.0f;
    for (int w = 0; w < kWarps; ++w) t += red[w][r];
    rinv[r] = rsqrtf(__fdividef(t, (float)d) + a.eps);
  }
  for (int c = threadIdx.x; c < nck; c += kThreads) {
    float g[8];
    if (a.norm_w) {
      row8<MMF_F32>(a.norm_w, 8 * c, g);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) g[e] = 1.0f;
    }
#pragma unroll
    for (int r = 0; r < NB; ++r) {
      float v[8];
      row8<XT>(a.x, (int64_t)r * d + 8 * c, v);
      // two planes of 4-value halves: lanes then read 16 consecutive bytes each, conflict-free
      float* lo = rs + (size_t)r * d + 4 * c;
      float* hi = lo + (d >> 1);
      *reinterpret_cast<float4*>(lo) = make_float4(v[0] * rinv[r] * g[0], v[1] * rinv[r] * g[1],
                                                   v[2] * rinv[r] * g[2], v[3] * rinv[r] * g[3]);
      *reinterpret_cast<float4*>(hi) = make_float4(v[4] * rinv[r] * g[4], v[5] * rinv[r] * g[5],
                                                   v[6] * rinv[r] * g[6], v[7] * rinv[r] * g[7]);
    }
  }
  __syncthreads();

  // 2. each warp takes VR vocabulary rows at a time (four from four token rows on: every shared-
  //    memory load of the normalised rows feeds 4x the FMAs and each step keeps 4 table rows of
  //    bytes in flight): 8 values per lane per step, float32 accumulation; the table words are
  //    unpacked where they are used, which keeps two CTAs per SM
  constexpr int VR = NB >= 4 ? 4 : 1;
  const int v0 = blockIdx.x * a.rows_per_cta;
  const int v1 = min(a.vocab, v0 + a.rows_per_cta);
  float best[NB];
  int bidx[NB];
#pragma unroll
  for (int r = 0; r < NB; ++r) { best[r] = -INFINITY; bidx[r] = 0x7fffffff; }
  for (int vb = v0 + warp * VR; vb < v1; vb += kWarps * VR) {
    float acc[VR][NB];
#pragma unroll
    for (int u = 0; u < VR; ++u)
#pragma unroll
      for (int r = 0; r < NB; ++r) acc[u][r] = 0.0f;
    // the table stream runs one chunk ahead: chunk c + 32's words are requested before chunk c
    // is multiplied
    Raw8h<TT> nxt[VR];
#pragma unroll
    for (int u = 0; u < VR; ++u)
      if (lane < nck && vb + u < v1) raw8h_load<TT>(a.table, (int64_t)(vb + u) * d + 8 * lane, nxt[u]);
    for (int c = lane; c < nck; c += 32) {
      Raw8h<TT> cur[VR];
#pragma unroll
      for (int u = 0; u < VR; ++u) {
        cur[u] = nxt[u];
        if (vb + u >= v1) cur[u] = Raw8h<TT>{};  // rows past the slice contribute zeros
      }
#pragma unroll
      for (int u = 0; u < VR; ++u)
        if (c + 32 < nck && vb + u < v1) raw8h_load<TT>(a.table, (int64_t)(vb + u) * d + 8 * (c + 32), nxt[u]);
#pragma unroll
      for (int r = 0; r < NB; ++r) {
        const float4 p = *reinterpret_cast<const float4*>(rs + (size_t)r * d + 4 * c);
        const float4 q = *reinterpret_cast<const float4*>(rs + (size_t)r * d + (d >> 1) + 4 * c);
#pragma unroll
        for (int u = 0; u < VR; ++u) {
          float e8[8];
          raw8h_unpack<TT>(cur[u], e8);
          acc[u][r] = fmaf(e8[0], p.x, acc[u][r]); acc[u][r] = fmaf(e8[1], p.y, acc[u][r]);
          acc[u][r] = fmaf(e8[2], p.z, acc[u][r]); acc[u][r] = fmaf(e8[3], p.w, acc[u][r]);
          acc[u][r] = fmaf(e8[4], q.x, acc[u][r]); acc[u][r] = fmaf(e8[5], q.y, acc[u][r]);
          acc[u][r] = fmaf(e8[6], q.z, acc[u][r]); acc[u][r] = fmaf(e8[7], q.w, acc[u][r]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < VR; ++u) {
      const int v = vb + u;
#pragma unroll
      for (int r = 0; r < NB; ++r) {
        const float t = warp_sum(acc[u][r]);
        if (v < v1) {
          if (lane == 0 && a.logits) a.logits[(int64_t)r * a.ld_logits + v] = t;
          if (head_better(t, v, best[r], bidx[r])) { best[r] = t; bidx[r] = v; }
        }
      }
    }
  }
  // 3. the CTA's best per token row
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < NB; ++r) { wbest[warp][r] = best[r]; wbidx[warp][r] = bidx[r]; }
  }
  __syncthreads();
  if (threadIdx.x < NB) {
    const int r = threadIdx.x;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int w = 0; w < kWarps; ++w)
      if (head_better(wbest[w][r], wbidx[w][r], bv, bi)) { bv = wbest[w][r]; bi = wbidx[w][r]; }
    a.pmax[(int64_t)blockIdx.x * kRows + r] = bv;
    a.pidx[(int64_t)blockIdx.x * kRows + r] = bi;
  }
}

// One warp per token row: the best of the CTAs' candidates (`ld` entries per CTA).
__global__ void __launch_bounds__(kThreads) head_argmax_kernel(const float* __restrict__ pmax,
                                                               const int32_t* __restrict__ pidx,
                                                               int nparts, int ld, int b, int32_t* __restrict__ ids) {
  const int r = blockIdx.x * kWarps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= b) return;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int p = lane; p < nparts; p += 32) {
    const float v = pmax[(int64_t)p * ld + r];
    const int i = pidx[(int64_t)p * ld + r];
    if (head_better(v, i, bv, bi)) { bv = v; bi = i; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (head_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
  }
  if (lane == 0) ids[r] = bi;
}

// ---------------------------------------------------------------------------------------------
// tensor-core form (bf16 table)
// ---------------------------------------------------------------------------------------------
// logits[v][j] = sum_k E[v][k] r[j][k] is a skinny GEMM: the table is the A operand (M = 128
// vocabulary rows per CTA, K-major), the normalised token rows the B operand, D float32 in tensor
// memory. The MMA takes bf16 operands, so each float32 row r enters as two bf16 rows, hi = bf16(r)
// and lo = bf16(r - hi), which together carry 16 significant bits; the two halves of D add up in
// the epilogue to the product with r up to ~2^-17 relative, the size of float32 accumulation error
// over d terms. One CTA = one vocabulary tile over all of K: a producer thread streams 64-wide
// k-blocks of the table tile and of the token rows into a 4-stage ring with TMA (128-byte swizzle),
// one thread issues four MMAs (K = 16 each) per k-block, then all four warps read D back (warp w
// owns TMEM lanes 32w..32w+31, i.e. one vocabulary row per thread), write the logits and reduce
// the (maximum, lowest index) per token row. Every wait is bounded.
constexpr int kTcRowsMax = 128;   // token rows per pass: N = 2 x 128 = 256, the MMA maximum
constexpr int kTcMinRows = 2;     // calls with fewer token rows take the CUDA-core form
constexpr int kTcBM = 128;        // vocabulary rows per CTA (MMA M)
constexpr int kTcBK = 64;         // bf16 per k-block: one 128-byte swizzle atom
constexpr int kTcUK = 16;         // K per kind::f16 instruction
constexpr int kTcStages = 4;
constexpr int kTcThreads = 128;
constexpr int kTcABytes = kTcBM * kTcBK * 2;   // 16 KB table tile per stage
constexpr int kTcBars = 2 * kTcStages + 2;

__host__ __device__ constexpr int tc_stage_bytes(int h) { return kTcABytes + 2 * h * kTcBK * 2; }
__host__ __device__ constexpr int tc_smem_bytes(int h) {
  return 1024 + kTcStages * tc_stage_bytes(h) + kTcBars * 8 + 16;
}

struct TcParams {
  CUtensorMap tmap;     // table [vocab][d] bf16, box 64 x 128, 128-byte swizzle
  CUtensorMap xmap;     // hi / lo rows [2h][d] bf16, box 64 x 2h, 128-byte swizzle
  int32_t nb;           // token rows of the pass
  int32_t h;            // hi rows at [0, h), lo rows at [h, 2h); nb <= h, h % 16 == 0
  int32_t num_kb;       // ceil(d / 64); the tail k-block reads zeros past d on both operands
  int32_t vocab;
  float* logits;        // nullable [nb][ld_logits]
  int64_t ld_logits;
  float* pmax;          // [gridDim][kTcRowsMax]
  int32_t* pidx;
  uint32_t tmem_cols;   // power of two >= max(32, 2h)
  uint32_t wait_limit_us;
};

// r = x / rms(x) * w for token row j = blockIdx.x of the pass, stored as bf16 rows hi (row j) and
// lo (row h + j); slots j >= nb get zero rows.
template <mmf_dtype XT>
__global__ void __launch_bounds__(kThreads) head_pack_kernel(const void* __restrict__ x, int d,
                                                             const float* __restrict__ norm_w, float eps,
                                                             int nb, int h, __nv_bfloat16* __restrict__ xs) {
  __shared__ float red[32];
  const int j = blockIdx.x, nck = d >> 3;
  uint4* hi = reinterpret_cast<uint4*>(xs + (size_t)j * d);
  uint4* lo = reinterpret_cast<uint4*>(xs + (size_t)(h + j) * d);
  if (j >= nb) {
    for (int c = threadIdx.x; c < nck; c += kThreads) { hi[c] = make_uint4(0, 0, 0, 0); lo[c] = make_uint4(0, 0, 0, 0); }
    return;
  }
  float ss = 0.0f;
  for (int c = threadIdx.x; c < nck; c += kThreads) {
    float v[8];
    row8<XT>(x, (int64_t)j * d + 8 * c, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
  }
  const float rinv = rsqrtf(__fdividef(block_sum(ss, red), (float)d) + eps);
  for (int c = threadIdx.x; c < nck; c += kThreads) {
    float v[8], g[8];
    row8<XT>(x, (int64_t)j * d + 8 * c, v);
    if (norm_w) {
      row8<MMF_F32>(norm_w, 8 * c, g);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) g[e] = 1.0f;
    }
    uint32_t wh[4], wl[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float r0 = v[2 * q] * rinv * g[2 * q], r1 = v[2 * q + 1] * rinv * g[2 * q + 1];
      const __nv_bfloat162 ph = __floats2bfloat162_rn(r0, r1);
      const float2 hf = __bfloat1622float2(ph);
      const __nv_bfloat162 pl = __floats2bfloat162_rn(r0 - hf.x, r1 - hf.y);
      wh[q] = *reinterpret_cast<const uint32_t*>(&ph);
      wl[q] = *reinterpret_cast<const uint32_t*>(&pl);
    }
    hi[c] = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    lo[c] = make_uint4(wl[0], wl[1], wl[2], wl[3]);
  }
}

__global__ void __launch_bounds__(kTcThreads) head_tc_kernel(const __grid_constant__ TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ float wbv[kTcThreads / 32][kTcRowsMax];
  __shared__ int wbi[kTcThreads / 32][kTcRowsMax];
  const int h = P.h, nb = P.nb, num_kb = P.num_kb;
  const int stage_bytes = tc_stage_bytes(h);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTcStages * stage_bytes);
  uint64_t* full = bars;                     // TMA -> MMA          (count 1 + tx bytes)
  uint64_t* empty = bars + kTcStages;        // MMA commit -> TMA   (count 1)
  uint64_t* accfull = bars + 2 * kTcStages;  // MMA commit -> epilogue
  uint64_t* drain = accfull + 1;             // MMA drain after an abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kTcBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int v0 = blockIdx.x * kTcBM;
  const uint32_t limit = P.wait_limit_us;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&P.tmap);
    tma_prefetch_desc(&P.xmap);
  }
  if (warp == 1) tmem_alloc(tmem_slot, P.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int kb = 0;
      for (; kb < num_kb; ++kb) {
        const int s = kb % kTcStages;
        const uint32_t ph = (uint32_t)(kb / kTcStages) & 1u;
        if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_flag)) break;
        uint8_t* st = smem + s * stage_bytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)stage_bytes);
        tma_load_2d(st, &P.tmap, kb * kTcBK, v0, &full[s]);
        tma_load_2d(st + kTcABytes, &P.xmap, kb * kTcBK, 0, &full[s]);
      }
      if (kb < num_kb) {
        // drain: the stages armed in the last kTcStages iterations must see their copies land
        for (int j = kb > kTcStages ? kb - kTcStages : 0; j < kb; ++j)
          mbar_wait_drain(&full[j % kTcStages], (uint32_t)(j / kTcStages) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // kind::f16: D float32 (bits 4-5 = 1), A and B bf16 (bits 7-9, 10-12 = 1), both K-major,
      // N >> 3 at bits 17-22, M >> 4 at bits 24-28
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(2 * h) >> 3 << 17) |
                             ((uint32_t)(kTcBM >> 4) << 24);
      int kb = 0;
      for (; kb < num_kb; ++kb) {
        const int s = kb % kTcStages;
        const uint32_t ph = (uint32_t)(kb / kTcStages) & 1u;
        if (!mbar_wait_bounded(&full[s], ph, limit, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * stage_bytes);
        const uint32_t b_addr = a_addr + kTcABytes;
#pragma unroll
        for (int kk = 0; kk < kTcBK / kTcUK; ++kk)
          tc_mma_bf16_ss(tmem, sw128_desc(a_addr + kk * kTcUK * 2), sw128_desc(b_addr + kk * kTcUK * 2), idesc,
                         (kb | kk) != 0 ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      if (kb == num_kb) {
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
    const int v = v0 + warp * 32 + lane;
    const bool valid = v < P.vocab;
    const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
    for (int c0 = 0; c0 < nb; c0 += 16) {
      uint32_t hv[16], lv[16];
      tmem_ld_32x32b_x16(taddr + (uint32_t)c0, hv);
      tmem_ld_32x32b_x16(taddr + (uint32_t)(h + c0), lv);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int j = c0 + e;
        if (j < nb) {  // uniform across the warp
          const float val = __uint_as_float(hv[e]) + __uint_as_float(lv[e]);
          if (valid && P.logits) P.logits[(int64_t)j * P.ld_logits + v] = val;
          float bv = valid ? val : -INFINITY;
          int bi = valid ? v : 0x7fffffff;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (head_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
          }
          if (lane == 0) { wbv[warp][j] = bv; wbi[warp][j] = bi; }
        }
      }
    }
  } else if (lane == 0) {
    for (int j = 0; j < nb; ++j) { wbv[warp][j] = -INFINITY; wbi[warp][j] = 0x7fffffff; }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, P.tmem_cols);
  if (threadIdx.x < nb) {
    const int j = threadIdx.x;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int w = 0; w < kTcThreads / 32; ++w)
      if (head_better(wbv[w][j], wbi[w][j], bv, bi)) { bv = wbv[w][j]; bi = wbi[w][j]; }
    P.pmax[(int64_t)blockIdx.x * kTcRowsMax + j] = bv;
    P.pidx[(int64_t)blockIdx.x * kTcRowsMax + j] = bi;
  }
}

}  // namespace head
}  // namespace mmf
