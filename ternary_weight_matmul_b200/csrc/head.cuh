// head.cuh -- K10: tied language-model head and greedy next token (generation).
//
// logits = RMSNorm(x) . E^T with E the embedding table [vocab][d] that the input embedding
// shares, then next = argmax (lowest index among equal maxima). Only the last position of each
// sequence is needed to generate, so this runs on a handful of token rows and streams the table
// once per call: an HBM-bound product, done on the CUDA cores. Every CTA normalises the (up to
// kRows) token rows into shared memory in float32; each warp then forms the logits of its
// vocabulary rows from 16-byte table loads with float32 accumulation and keeps a running
// (maximum, lowest index) per token row; the CTA's best per row goes to a partial array that a
// one-warp-per-row kernel reduces to the ids.
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

// One warp per token row: the best of the CTAs' candidates.
__global__ void __launch_bounds__(kThreads) head_argmax_kernel(const float* __restrict__ pmax,
                                                               const int32_t* __restrict__ pidx,
                                                               int nparts, int b, int32_t* __restrict__ ids) {
  const int r = blockIdx.x * kWarps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= b) return;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int p = lane; p < nparts; p += 32) {
    const float v = pmax[(int64_t)p * kRows + r];
    const int i = pidx[(int64_t)p * kRows + r];
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

}  // namespace head
}  // namespace mmf
