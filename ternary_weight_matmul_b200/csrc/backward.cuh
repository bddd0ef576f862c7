// backward.cuh -- gradients of the HGRN recurrence with its gates, for a training step.
//
// Forward (the scan with fused gates): f = sigmoid(zf), i = SiLU(zi) (1 - f),
// h_t = f_t h_{t-1} + i_t. Given dL/dh_t for every step, the total gradient reaching h_t is
// G_t = dh_t + f_{t+1} G_{t+1}, taken backwards in time; then dL/di_t = G_t, dL/df_t = G_t h_{t-1},
// and through the gates dzf = (df - di SiLU(zi)) f (1 - f), dzi = di (1 - f) SiLU'(zi) with
// SiLU'(z) = sigmoid(z) (1 + z (1 - sigmoid(z))); dL/dh0 = f_0 G_0. The MatMul-Free LLM report
// (nightvoyager.top, innovations table) names the straight-through estimator for training; the
// recurrence and its gates are smooth, so these are their exact derivatives.
//
// G obeys the affine recurrence G_t = f_{t+1} G_{t+1} + dh_t backwards in time, so it is chunked
// like the forward scan with the time axis reversed. With `carry` = f_{t1} G_{t1}, what enters
// chunk [t0, t1) from the later steps (0 for the last chunk), the chunk passes f_{t0} G_{t0} =
// A carry + B on to the earlier steps, A the product of its forget gates and B the value at
// carry 0. Phase 1 folds every (sequence, chunk, channel) into (A, B) reading zf and dh; phase 2
// walks the chunks of each channel from the last to the first and records every chunk's carry
// (the final one is dh0); phase 3 replays each chunk from its carry, reading zf, zi, dh and
// h_{t-1} and writing dzf and dzi. Sequences no longer than one chunk take phase 3 alone. Each
// thread owns VEC adjacent channels (paired loads when rows allow), lanes cover consecutive
// channels, so every access is a coalesced row segment; steps are loaded ahead into registers
// before the dependent chain runs over them.
// FusedBitLinear with the straight-through estimator (the report: weight_quant quantises in the
// forward pass and keeps the gradient in the backward pass; the activation quantiser is taken the
// same way): with the forward's codes q and factors a/127, the dequantised operands are
// rq = q (a/127) and Wq = t s, and
//   dr = dy Wq;  u = dr w;  rho = (mean(x^2) + eps)^(-1/2);  dx = rho u - rho^3 x mean(u x);
//   dw[k] = sum_m dr[m][k] x[m][k] rho_m;  dW = dy^T rq  (the latent weight's gradient).
// dr and dW are products: on the tensor cores (bf16_gemm_kernel, with the operand layout kernels
// below) or, on the CUDA-core engine, one thread per (row, 16-column word of the packed codes)
// for dr and per (weight row, column) for dW. dr is written into dx's buffer; one row-block
// kernel then forms rho, the gain's gradient partials and dx in place over dr.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"

namespace mmf {
namespace bwd {

constexpr int kThreads = 256;

struct ScanBwdArgs {
  const void* zf;     // [b][t][d] pre-activations of the forget gate
  const void* zi;     // [b][t][d] pre-activations of the input
  const void* h;      // [b][t][d] forward states
  const void* dh;     // [b][t][d] dL/dh_t
  mmf_dtype dt;       // of zf, zi, h, dh, dzf, dzi
  int32_t b;
  int64_t t;
  int32_t d;
  const float* h0;    // [b][d] or null (zeros)
  void* dzf;          // [b][t][d] out
  void* dzi;          // [b][t][d] out
  float* dh0;         // [b][d] out, or null
  int32_t chunk;      // steps per chunk
  int32_t nchunk;
  int32_t gx;         // CTAs across the channels of one (sequence, chunk)
  float* agg_a;       // [b][nchunk][d] product of the chunk's forget gates
  float* agg_b;       // [b][nchunk][d] f_{t0} G_{t0} of the chunk at carry 0
  float* cin;         // [b][nchunk][d] carry entering each chunk from the later steps
};
constexpr int kScanBwdThreads = 128;
constexpr int kScanBwdFold = 8;     // steps loaded ahead in phase 1 (two arrays)
constexpr int kScanBwdReplay = 4;   // steps loaded ahead in phase 3 (four arrays)

// Steps are loaded ahead as raw words (a bf16 pair in one register) and widened to float32 only
// when used, which keeps the prefetch to one register per bf16 value pair.
template <mmf_dtype DT, int VEC>
struct RawV {
  using T = typename std::conditional<DT == MMF_F32 && VEC == 2, uint2, uint32_t>::type;
};
template <mmf_dtype DT, int VEC>
__device__ __forceinline__ typename RawV<DT, VEC>::T raw_load(const void* base, int64_t idx) {
  if constexpr (DT == MMF_F32 && VEC == 2) {
    return *reinterpret_cast<const uint2*>(reinterpret_cast<const float*>(base) + idx);
  } else if constexpr (DT == MMF_F32) {
    return *reinterpret_cast<const uint32_t*>(reinterpret_cast<const float*>(base) + idx);
  } else if constexpr (VEC == 2) {
    return *reinterpret_cast<const uint32_t*>(reinterpret_cast<const __nv_bfloat16*>(base) + idx);
  } else {
    return (uint32_t)*reinterpret_cast<const unsigned short*>(reinterpret_cast<const __nv_bfloat16*>(base) + idx);
  }
}
template <mmf_dtype DT, int VEC>
__device__ __forceinline__ void raw_unpack(const typename RawV<DT, VEC>::T& r, float (&o)[VEC]) {
  if constexpr (DT == MMF_F32 && VEC == 2) {
    o[0] = __uint_as_float(r.x);
    o[VEC - 1] = __uint_as_float(r.y);
  } else if constexpr (DT == MMF_F32) {
    o[0] = __uint_as_float(r);
  } else if constexpr (VEC == 2) {
    o[0] = __uint_as_float(r << 16);
    o[VEC - 1] = __uint_as_float(r & 0xffff0000u);
  } else {
    o[0] = __uint_as_float(r << 16);
  }
}

// blockIdx.x runs over (sequence, chunk, channel block) with the channel block fastest, so the
// grid has no per-dimension limit on b or the chunk count.
__device__ __forceinline__ void scan_bwd_block(const ScanBwdArgs& a, int& cx, int& c, int& bi) {
  const int64_t id = blockIdx.x;
  const int64_t rest = id / a.gx;
  cx = (int)(id - rest * a.gx);
  bi = (int)(rest / a.nchunk);
  c = (int)(rest - (int64_t)bi * a.nchunk);
}

// Phase 1: (A, B) of every (sequence, chunk, channel).
template <mmf_dtype DT, int VEC>
__global__ void __launch_bounds__(kScanBwdThreads) scan_bwd_fold_kernel(const ScanBwdArgs a) {
  int cx, c, bi;
  scan_bwd_block(a, cx, c, bi);
  const int64_t ch = ((int64_t)cx * kScanBwdThreads + threadIdx.x) * VEC;
  if (ch >= a.d) return;
  const int64_t t0 = (int64_t)c * a.chunk;
  const int64_t t1 = t0 + a.chunk < a.t ? t0 + a.chunk : a.t;
  const int64_t base = (int64_t)bi * a.t * a.d + ch;
  float A[VEC], B[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) { A[v] = 1.0f; B[v] = 0.0f; }
  using R = typename RawV<DT, VEC>::T;
  for (int64_t te = t1; te > t0; te -= kScanBwdFold) {
    R rzf[kScanBwdFold], rdh[kScanBwdFold];
#pragma unroll
    for (int u = 0; u < kScanBwdFold; ++u) {
      if (te - 1 - u >= t0) {
        rzf[u] = raw_load<DT, VEC>(a.zf, base + (te - 1 - u) * a.d);
        rdh[u] = raw_load<DT, VEC>(a.dh, base + (te - 1 - u) * a.d);
      }
    }
#pragma unroll
    for (int u = 0; u < kScanBwdFold; ++u) {
      if (te - 1 - u >= t0) {
        float zf[VEC], dh[VEC];
        raw_unpack<DT, VEC>(rzf[u], zf);
        raw_unpack<DT, VEC>(rdh[u], dh);
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
          float f, omf;
          hgrn_forget(zf[v], f, omf);
          B[v] = f * (dh[v] + B[v]);
          A[v] = f * A[v];
        }
      }
    }
  }
  const int64_t o = ((int64_t)bi * a.nchunk + c) * a.d + ch;
#pragma unroll
  for (int v = 0; v < VEC; ++v) {
    a.agg_a[o + v] = A[v];
    a.agg_b[o + v] = B[v];
  }
}

// Phase 2: one thread per (sequence, channel) walks the chunks from the last to the first.
__global__ void __launch_bounds__(kScanBwdThreads) scan_bwd_carry_kernel(const ScanBwdArgs a) {
  const int64_t gid = (int64_t)blockIdx.x * kScanBwdThreads + threadIdx.x;
  if (gid >= (int64_t)a.b * a.d) return;
  const int bi = (int)(gid / a.d);
  const int64_t ch = gid - (int64_t)bi * a.d;
  const int64_t base = (int64_t)bi * a.nchunk * a.d + ch;
  float carry = 0.0f;
  constexpr int PF = 32;
  for (int c1 = a.nchunk; c1 > 0; c1 -= PF) {
    float av[PF], bv[PF];
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      if (c1 - 1 - u >= 0) {
        av[u] = a.agg_a[base + (int64_t)(c1 - 1 - u) * a.d];
        bv[u] = a.agg_b[base + (int64_t)(c1 - 1 - u) * a.d];
      }
    }
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      if (c1 - 1 - u >= 0) {
        a.cin[base + (int64_t)(c1 - 1 - u) * a.d] = carry;
        carry = fmaf(av[u], carry, bv[u]);
      }
    }
  }
  if (a.dh0) a.dh0[gid] = carry;
}

// Phase 3: replays chunk c from its carry and writes dzf, dzi; with SINGLE the sequence is one
// chunk entered with carry 0, and its f_0 G_0 is dh0.
template <mmf_dtype DT, int VEC, bool SINGLE>
__global__ void __launch_bounds__(kScanBwdThreads) scan_bwd_replay_kernel(const ScanBwdArgs a) {
  int cx, c, bi;
  scan_bwd_block(a, cx, c, bi);
  const int64_t ch = ((int64_t)cx * kScanBwdThreads + threadIdx.x) * VEC;
  if (ch >= a.d) return;
  const int64_t t0 = (int64_t)c * a.chunk;
  const int64_t t1 = t0 + a.chunk < a.t ? t0 + a.chunk : a.t;
  const int64_t base = (int64_t)bi * a.t * a.d + ch;
  float cterm[VEC], hinit[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) {
    cterm[v] = SINGLE ? 0.0f : a.cin[((int64_t)bi * a.nchunk + c) * a.d + ch + v];
    hinit[v] = a.h0 ? a.h0[(int64_t)bi * a.d + ch + v] : 0.0f;
  }
  using R = typename RawV<DT, VEC>::T;
  for (int64_t te = t1; te > t0; te -= kScanBwdReplay) {
    R rzf[kScanBwdReplay], rzi[kScanBwdReplay], rdh[kScanBwdReplay], rhp[kScanBwdReplay];
#pragma unroll
    for (int u = 0; u < kScanBwdReplay; ++u) {
      const int64_t t = te - 1 - u;
      if (t >= t0) {
        rzf[u] = raw_load<DT, VEC>(a.zf, base + t * a.d);
        rzi[u] = raw_load<DT, VEC>(a.zi, base + t * a.d);
        rdh[u] = raw_load<DT, VEC>(a.dh, base + t * a.d);
        if (t > 0) rhp[u] = raw_load<DT, VEC>(a.h, base + (t - 1) * a.d);
      }
    }
#pragma unroll
    for (int u = 0; u < kScanBwdReplay; ++u) {
      const int64_t t = te - 1 - u;
      if (t >= t0) {
        float zf[VEC], zi[VEC], dh[VEC], hp[VEC];
        raw_unpack<DT, VEC>(rzf[u], zf);
        raw_unpack<DT, VEC>(rzi[u], zi);
        raw_unpack<DT, VEC>(rdh[u], dh);
        if (t > 0) {
          raw_unpack<DT, VEC>(rhp[u], hp);
        } else {
#pragma unroll
          for (int v = 0; v < VEC; ++v) hp[v] = hinit[v];
        }
        float gzf[VEC], gzi[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
          const float G = dh[v] + cterm[v];
          float f, omf;
          hgrn_forget(zf[v], f, omf);
          const float z = zi[v];
          const float sz = sigmoidf_(z);
          gzf[v] = (G * hp[v] - G * (z * sz)) * f * omf;
          gzi[v] = G * omf * sz * fmaf(z, 1.0f - sz, 1.0f);
          cterm[v] = f * G;
        }
        store_vec<DT, VEC>(a.dzf, base + t * a.d, gzf);
        store_vec<DT, VEC>(a.dzi, base + t * a.d, gzi);
      }
    }
  }
  if (SINGLE && a.dh0) {
#pragma unroll
    for (int v = 0; v < VEC; ++v) a.dh0[(int64_t)bi * a.d + ch + v] = cterm[v];
  }
}


struct LinBwdArgs {
  const void* x;        // [m][k] xdt
  mmf_dtype xdt;
  int64_t m;
  int32_t k;
  int32_t n;
  const float* norm_w;  // [k] or null (unit gain)
  float eps;
  const uint32_t* codes;  // [n][kw] packed ternary codes
  int32_t kw;
  const float* scale;   // 1 float
  const int8_t* q;      // [m][k] the forward's activation codes
  const float* deq;     // [m] the forward's a/127
  const void* dy;       // [m][n] dydt
  mmf_dtype dydt;
  float* dx;            // [m][k]: dr first, then dx
  float* dnorm_w;       // [k] or null
  float* dW;            // [n][k] or null
  float* rho;           // [m] scratch
};

// dr[m][16 w + j] = s sum_n dy[m][n] t[n][16 w + j]: one thread per (row, packed word column w),
// the 16 codes of word (n, w) expanded to int8 lanes (quad q = columns 4q..4q+3, lowest column in
// byte 0).
__global__ void __launch_bounds__(kThreads) lin_bwd_dr_kernel(const LinBwdArgs a) {
  const int w = blockIdx.y * kThreads + threadIdx.x;
  const int64_t row = blockIdx.x;
  if (w * 16 >= a.k) return;
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
  for (int nn = 0; nn < a.n; ++nn) {
    const float g = load_as_float(a.dy, row * a.n + nn, a.dydt);
    uint32_t quads[4];
    expand_word(a.codes[(int64_t)nn * a.kw + w], quads);
#pragma unroll
    for (int qd = 0; qd < 4; ++qd)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[4 * qd + e] = fmaf(g, (float)(int8_t)(quads[qd] >> (8 * e)), acc[4 * qd + e]);
  }
  const float s = *a.scale;
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if (16 * w + j < a.k) a.dx[row * a.k + 16 * w + j] = acc[j] * s;
}

// rho, the gain's gradient and dx for a block of rows_per rows (blockIdx.x), in one kernel:
// phase A, one warp per row: rho_r = (mean(x^2) + eps)^(-1/2) and mean(u x) with u = dr w (into
// rho[] and mux[]); phase B, threads over columns walking the block's rows in order:
// part[block][c] = sum_r dr x rho (before dx replaces dr), then dx = rho u - rho^3 x mean(u x) in
// place over dr. The partials are added per column by lin_bwd_dnw_reduce_kernel.
__global__ void __launch_bounds__(kThreads) lin_bwd_rows_kernel(const LinBwdArgs a, float* mux, float* part,
                                                                int rows_per) {
  const int64_t r0 = (int64_t)blockIdx.x * rows_per;
  const int64_t r1 = r0 + rows_per < a.m ? r0 + rows_per : a.m;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t r = r0 + warp; r < r1; r += kThreads / 32) {
    float ss = 0.0f, ux = 0.0f;
    for (int c = lane; c < a.k; c += 32) {
      const float xv = load_as_float(a.x, r * a.k + c, a.xdt);
      const float u = a.dx[r * a.k + c] * (a.norm_w ? a.norm_w[c] : 1.0f);
      ss = fmaf(xv, xv, ss);
      ux = fmaf(u, xv, ux);
    }
    ss = warp_sum(ss);
    ux = warp_sum(ux);
    if (lane == 0) {
      a.rho[r] = rsqrtf(ss / (float)a.k + a.eps);
      mux[r] = ux / (float)a.k;
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < a.k; c += kThreads) {
    const float w = a.norm_w ? a.norm_w[c] : 1.0f;
    float acc = 0.0f;
    for (int64_t rb = r0; rb < r1; rb += 4) {
      // four rows' loads in flight before the (ordered) arithmetic
      float d[4], xv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (rb + u < r1) {
          d[u] = a.dx[(rb + u) * a.k + c];
          xv[u] = load_as_float(a.x, (rb + u) * a.k + c, a.xdt);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (rb + u < r1) {
          const int64_t r = rb + u;
          const float rho = a.rho[r];
          acc = fmaf(d[u] * xv[u], rho, acc);
          a.dx[r * a.k + c] = rho * (d[u] * w) - rho * rho * rho * xv[u] * mux[r];
        }
      }
    }
    if (part) part[(int64_t)blockIdx.x * a.k + c] = acc;
  }
}
// dw[c] = sum over blocks of part[block][c], in block order; 32 columns x 8 lanes per CTA, each
// lane adding every 8th block, then the 8 lane sums in order.
__global__ void __launch_bounds__(256) lin_bwd_dnw_reduce_kernel(const LinBwdArgs a, const float* part, int splits) {
  __shared__ float red[8][33];
  const int c = blockIdx.x * 32 + threadIdx.x;
  float t = 0.0f;
  if (c < a.k)
    for (int z = threadIdx.y; z < splits; z += 8) t += part[(int64_t)z * a.k + c];
  red[threadIdx.y][threadIdx.x] = t;
  __syncthreads();
  if (threadIdx.y == 0 && c < a.k) {
    float s = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) s += red[j][threadIdx.x];
    a.dnorm_w[c] = s;
  }
}

// dW[n][c] = sum_m dy[m][n] q[m][c] (a/127)_m, one thread per (weight row, column); m = 0 gives
// zeros.
__global__ void __launch_bounds__(kThreads) lin_bwd_dw_kernel(const LinBwdArgs a) {
  const int c = blockIdx.x * kThreads + threadIdx.x;
  const int nn = blockIdx.y;
  if (c >= a.k) return;
  float acc = 0.0f;
  for (int64_t row = 0; row < a.m; ++row)
    acc = fmaf(load_as_float(a.dy, row * a.n + nn, a.dydt) * a.deq[row], (float)a.q[row * a.k + c], acc);
  a.dW[(int64_t)nn * a.k + c] = acc;
}

// Operands of the tensor-core form of dr and dW (bf16_gemm_kernel): bf16 arrays, K-major, row
// pitch ld (a multiple of 8 elements). A float32 value v enters as hi = bf16(v) and
// lo = bf16(v - hi); the codes are exact in bf16.
__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16* hi, __nv_bfloat16* lo, int64_t idx) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  hi[idx] = h;
  if (lo) lo[idx] = __float2bfloat16_rn(v - __bfloat162float(h));
}

// dr's A operand: dy [m][n] as hi / lo rows [m][ld].
__global__ void __launch_bounds__(kThreads) lin_bwd_split_kernel(const LinBwdArgs a, __nv_bfloat16* hi,
                                                                 __nv_bfloat16* lo, int64_t ld) {
  const int64_t total = a.m * a.n;
  for (int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x; e < total; e += (int64_t)gridDim.x * kThreads) {
    const int64_t r = e / a.n, c = e - r * a.n;
    split_bf16(load_as_float(a.dy, e, a.dydt), hi, lo, r * ld + c);
  }
}

// Transposed operands, dst[c][r] = value(r, c), through 32 x 32 shared-memory tiles (block 32 x 8;
// blockIdx.x over rows r, blockIdx.y over columns c):
//   kTrDyScaled  dW's A:  r = token, c = output feature: dy[r][c] * (a/127)_r as hi / lo   [n][ld]
//   kTrCodes     dW's B:  r = token, c = input feature:  q[r][c]                            [k][ld]
//   kTrTernary   dr's B:  r = weight row, c = input feature: t[r][c] from the packed words   [k][ld]
enum TrMode : int { kTrDyScaled = 0, kTrCodes = 1, kTrTernary = 2 };

template <int MODE>
__global__ void __launch_bounds__(256) lin_bwd_transpose_kernel(const LinBwdArgs a, __nv_bfloat16* hi,
                                                                __nv_bfloat16* lo, int64_t ld) {
  __shared__ float tile[32][33];
  const int64_t rows = MODE == kTrTernary ? (int64_t)a.n : a.m;
  const int cols = MODE == kTrDyScaled ? a.n : a.k;
  const int64_t r0 = (int64_t)blockIdx.x * 32;
  const int c0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int j = ty; j < 32; j += 8) {
    const int64_t r = r0 + j;
    const int c = c0 + tx;
    float v = 0.0f;
    if (r < rows && c < cols) {
      if (MODE == kTrDyScaled) {
        v = load_as_float(a.dy, r * a.n + c, a.dydt) * a.deq[r];
      } else if (MODE == kTrCodes) {
        v = (float)a.q[r * a.k + c];
      } else {
        const uint32_t word = a.codes[r * a.kw + (c >> 4)];
        const int jj = c & 15, quad = jj >> 2, ln = jj & 3;
        const uint32_t f = (word >> (16 * (quad >> 1) + 2 * (quad & 1) + 4 * ln)) & 3u;
        v = f == 1u ? 1.0f : (f == 3u ? -1.0f : 0.0f);
      }
    }
    tile[j][tx] = v;
  }
  __syncthreads();
  for (int j = ty; j < 32; j += 8) {
    const int c = c0 + j;
    const int64_t r = r0 + tx;
    if (c < cols && r < rows) split_bf16(tile[tx][j], hi, MODE == kTrDyScaled ? lo : nullptr, (int64_t)c * ld + r);
  }
}

}  // namespace bwd
}  // namespace mmf
