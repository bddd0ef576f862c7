// kernels.cuh -- CUDA-core kernels of libmmf: ternary weight packing, fused RMSNorm + int8
// quantisation (with the GLU and g_norm producers fused in front), the CUDA-core ternary GEMM for
// few rows, the HGRN scan and the embedding gather.
#pragma once

#include "common.cuh"

namespace mmf {

// =============================================================================================
// K0: weight_quant + 2-bit packing
// =============================================================================================
constexpr int kPackSumBlocks = 296;  // fixed grid for a deterministic float64 sum

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Partial sums of |W| in float64, one per block, fixed order.
template <mmf_dtype WT>
__global__ void __launch_bounds__(256) pack_abssum_kernel(const typename Elem<WT>::T* __restrict__ w,
                                                          int64_t count, double* __restrict__ partial) {
  __shared__ double red[8];
  double s = 0.0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x)
    s += fabs((double)Elem<WT>::load(w + i));
  s = warp_sum_d(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double r = threadIdx.x < 8 ? red[threadIdx.x] : 0.0;
    r = warp_sum_d(r);
    if (threadIdx.x == 0) partial[blockIdx.x] = r;
  }
}

// s = max(sum / count, 1e-5) as float32.
__global__ void __launch_bounds__(32) pack_scale_kernel(const double* __restrict__ partial, int nparts,
                                                        int64_t count, float* __restrict__ scale_out) {
  double s = 0.0;
  for (int i = threadIdx.x; i < nparts; i += 32) s += partial[i];
  s = warp_sum_d(s);
  if (threadIdx.x == 0) {
    double mean = count > 0 ? s / (double)count : 0.0;
    scale_out[0] = (float)fmax(mean, 1e-5);
  }
}

// One thread per packed word: codes clamp(rint(w / s), -1, 1) in float32, placed at the
// documented bit offsets; columns >= k are zero codes.
template <mmf_dtype WT>
__global__ void __launch_bounds__(256) pack_codes_kernel(const typename Elem<WT>::T* __restrict__ w,
                                                         int32_t n, int32_t k, int32_t kw,
                                                         const float* __restrict__ scale,
                                                         uint32_t* __restrict__ codes) {
  const int64_t total = (int64_t)n * kw;
  const float s = scale[0];
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = idx / kw;
    const int32_t wi = (int32_t)(idx - row * kw);
    uint32_t word = 0u;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int32_t col = wi * 16 + j;
      if (col < k) {
        const float v = __fdiv_rn(Elem<WT>::load(w + row * k + col), s);
        const float r = fminf(fmaxf(rintf(v), -1.0f), 1.0f);
        const uint32_t field = r > 0.5f ? 1u : (r < -0.5f ? 3u : 0u);
        const int quad = j >> 2, lane = j & 3;
        word |= field << (16 * (quad >> 1) + 2 * (quad & 1) + 4 * lane);
      }
    }
    codes[idx] = word;
  }
}

// =============================================================================================
// K1 / K5: fused row producer + RMSNorm + per-token absmax int8 quantisation
// =============================================================================================
enum RowMode : int {
  kRowPlain = 0,  // v = x[m][k]
  kRowGlu = 1,    // v = SiLU(x[m][k]) * x[m][k + K]        (x rows hold [gate | up])
  kRowGnorm = 2   // v = h[m][k] / rms(h[m]) * gw[k] * SiLU(g[m][k])   (g_norm output)
};

struct NormQuantArgs {
  const void* x;   // plain: x; glu: [gate|up]; gnorm: h
  int64_t ldx;
  mmf_dtype xdt;
  const void* g;   // gnorm: g (dtype gdt)
  int64_t ldg;
  mmf_dtype gdt;
  const float* gw; // gnorm gain (nullable = 1)
  int64_t m;
  int32_t k;       // features of v
  float eps;
  int32_t ngain;   // 1..3 independent norm gains sharing the rms of v
  const float* gain[3];
  int8_t* q[3];    // [m][ldq] (columns [k, ldq) are written as 0)
  int64_t ldq;
  float* deq[3];   // [m]
  int32_t pre_act; // 1: the SiLU of the gate input (g for g_norm, the gate half for GLU) is precomputed
};

// 1 / sqrt(ss / k + eps) in float32 (approximate reciprocal square root: 1/rms is a common
// factor of a row's values and of their maximum, so it reaches a code only through rounding).
__device__ __forceinline__ float nq_rinv(float ss, int k, float eps) {
  return rsqrtf(__fdividef(ss, (float)k) + eps);
}
// 127 / a (correctly rounded: it sets every code of the row) and a / 127 (the dequantisation
// factor, within 1.5 ulp), for a >= 1e-5.
__device__ __forceinline__ float q127_over(float a) { return __fdiv_rn(127.0f, a); }
__device__ __forceinline__ float over_127(float a) { return a * (1.0f / 127.0f); }

__device__ __forceinline__ double block_sum_d(double v, double* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum_d(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  double r = lane < nw ? red[lane] : 0.0;
  return warp_sum_d(r);
}

// One CTA per row; v is materialised once in shared memory (k floats). The mean square and the
// normalised value r = v / sqrt(ms + eps) * gain are formed in float64 and rounded once to
// float32, so the int8 decision rint(r * 127/a) (float32) sees the correctly rounded r.
template <int MODE>
__global__ void __launch_bounds__(256) norm_quant_kernel(const NormQuantArgs a) {
  extern __shared__ float vrow[];
  __shared__ double redd[32];
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const int k = a.k;
  double rinv_h = 1.0;
  if (MODE == kRowGnorm) {
    double ss = 0.0;
    for (int c = threadIdx.x; c < k; c += blockDim.x) {
      const double hv = load_as_float(a.x, row * a.ldx + c, a.xdt);
      ss += hv * hv;
    }
    ss = block_sum_d(ss, redd);
    rinv_h = 1.0 / sqrt(ss / (double)k + (double)a.eps);
  }
  double ss = 0.0;
  for (int c = threadIdx.x; c < k; c += blockDim.x) {
    float v;
    if (MODE == kRowPlain) {
      v = load_as_float(a.x, row * a.ldx + c, a.xdt);
    } else if (MODE == kRowGlu) {
      const float gate = load_as_float(a.x, row * a.ldx + c, a.xdt);
      const float up = load_as_float(a.x, row * a.ldx + k + c, a.xdt);
      v = (a.pre_act ? gate : siluf_(gate)) * up;
    } else {
      const double hv = load_as_float(a.x, row * a.ldx + c, a.xdt);
      const float gv = load_as_float(a.g, row * a.ldg + c, a.gdt);
      v = (float)(hv * rinv_h * (double)(a.gw ? a.gw[c] : 1.0f)) * (a.pre_act ? gv : siluf_(gv));
    }
    vrow[c] = v;
    ss += (double)v * (double)v;
  }
  ss = block_sum_d(ss, redd);
  const double rinv = 1.0 / sqrt(ss / (double)k + (double)a.eps);
  for (int j = 0; j < a.ngain; ++j) {
    const float* gn = a.gain[j];
    float amax = 0.0f;
    for (int c = threadIdx.x; c < k; c += blockDim.x) {
      const float r = (float)((double)vrow[c] * rinv * (double)(gn ? gn[c] : 1.0f));
      amax = fmaxf(amax, fabsf(r));
    }
    amax = fmaxf(block_max(amax, red), 1e-5f);
    const float sx = q127_over(amax);
    int8_t* qrow = a.q[j] + row * a.ldq;
    for (int c = threadIdx.x; c < a.ldq; c += blockDim.x) {
      int8_t code = 0;
      if (c < k) {
        const float r = (float)((double)vrow[c] * rinv * (double)(gn ? gn[c] : 1.0f));
        code = (int8_t)fminf(fmaxf(rintf(__fmul_rn(r, sx)), -127.0f), 127.0f);
      }
      qrow[c] = code;
    }
    if (threadIdx.x == 0) a.deq[j][row] = over_127(amax);
  }
}

// Vectorised variant for K % 8 == 0 and 16-byte aligned rows (K <= 8192): a row group of W
// warps owns one row and keeps it in registers (NCH chunks of 8 values per thread), loads and
// stores whole 16-/8-byte pieces and reduces with shuffles (plus one double-buffered shared
// exchange per reduction when W > 1). NG is 1 or 3 norm gains sharing the row's rms.
//
// Arithmetic: r = (v * (1/rms)) * gain in float32, a = max|r|, code = rint(r * (127/a)). The
// factor 1/rms cancels between r and a, so the codes depend on the mean square only through the
// float32 rounding of r (a relative perturbation of the mean square moves r * 127/a by a few
// ulp at most); the sum of squares and 1/sqrt therefore run in float32 (each step IEEE-rounded).
// The dequantisation factor a/127 carries the mean square's own rounding (~1e-7 relative).
constexpr int kNqThreads = 128;

template <int W>
__device__ __forceinline__ float nq_group_sum(float v, float (*red)[8], int& ph) {
  v = warp_sum(v);
  if (W == 1) return v;
  const int wid = threadIdx.x >> 5, g0 = (wid / W) * W;
  float* r = red[ph & 1];
  ++ph;
  if ((threadIdx.x & 31) == 0) r[wid] = v;
  __syncthreads();
  float s = 0.0f;
#pragma unroll
  for (int k = 0; k < W; ++k) s += r[g0 + k];
  return s;
}
// Maxima of NG values over the row group (one exchange for all gains).
template <int W, int NG>
__device__ __forceinline__ void nq_group_max(float (&v)[NG], float (*red)[8][3], int& ph) {
#pragma unroll
  for (int j = 0; j < NG; ++j) v[j] = warp_max(v[j]);
  if (W == 1) return;
  const int wid = threadIdx.x >> 5, g0 = (wid / W) * W;
  float(*r)[3] = red[ph & 1];
  ++ph;
  if ((threadIdx.x & 31) == 0) {
#pragma unroll
    for (int j = 0; j < NG; ++j) r[wid][j] = v[j];
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < NG; ++j) {
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < W; ++k) m = fmaxf(m, r[g0 + k][j]);
    v[j] = m;
  }
}

template <mmf_dtype DT>
__device__ __forceinline__ void load8(const void* base, int64_t idx, float (&o)[8]) {
  if (DT == MMF_BF16) {
    const uint4 u = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(base) + idx);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[q]));
      o[2 * q] = f.x;
      o[2 * q + 1] = f.y;
    }
  } else {
    const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx);
    const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx + 4);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  }
}
// Bits of x + 1.5 * 2^23 for |x| < 127.5: the addition (where the float32 spacing is exactly 1)
// rounds half to even, and the low byte of the result is the int8 code rint(x) itself
// (0x4B400000 has a zero low byte). No clamp is needed: x = r * fl(127 / a) with a the maximum of
// the very |r| values, so |x| <= 127 (1 + 2^-24)^2 < 127.5 and the code lies in [-127, 127].
__device__ __forceinline__ uint32_t q8_bits(float x) { return __float_as_uint(__fadd_rn(x, 12582912.0f)); }
__device__ __forceinline__ float2 q8_add2(float2 x) {
  return __fadd2_rn(x, make_float2(12582912.0f, 12582912.0f));
}
// Low bytes of four words packed into one word, a in byte 0.
__device__ __forceinline__ uint32_t pack4_lo_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x0040u), 0x5410u);
}
// Eight codes (four float2 of x + 1.5 * 2^23) as two words.
__device__ __forceinline__ uint2 pack8_codes(const float2 (&b)[4]) {
  return make_uint2(pack4_lo_bytes(__float_as_uint(b[0].x), __float_as_uint(b[0].y), __float_as_uint(b[1].x),
                                   __float_as_uint(b[1].y)),
                    pack4_lo_bytes(__float_as_uint(b[2].x), __float_as_uint(b[2].y), __float_as_uint(b[3].x),
                                   __float_as_uint(b[3].y)));
}

// Raw 8-value chunks (one 16-byte word for bf16, two for float32), loaded a row ahead of use.
template <mmf_dtype XT> struct Raw8 { uint4 w[XT == MMF_F32 ? 2 : 1]; };
template <mmf_dtype XT>
__device__ __forceinline__ void raw8_load(const void* base, int64_t idx, Raw8<XT>& r) {
  const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(base) + idx * (XT == MMF_F32 ? 4 : 2));
  r.w[0] = __ldcs(p);
  if (XT == MMF_F32) r.w[XT == MMF_F32 ? 1 : 0] = __ldcs(p + 1);
}
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
template <mmf_dtype XT>
__device__ __forceinline__ void raw8_unpack(const Raw8<XT>& r, float2 (&o)[4]) {
  if (XT == MMF_F32) {
    o[0] = make_float2(__uint_as_float(r.w[0].x), __uint_as_float(r.w[0].y));
    o[1] = make_float2(__uint_as_float(r.w[0].z), __uint_as_float(r.w[0].w));
    o[2] = make_float2(__uint_as_float(r.w[XT == MMF_F32 ? 1 : 0].x), __uint_as_float(r.w[XT == MMF_F32 ? 1 : 0].y));
    o[3] = make_float2(__uint_as_float(r.w[XT == MMF_F32 ? 1 : 0].z), __uint_as_float(r.w[XT == MMF_F32 ? 1 : 0].w));
  } else {
    o[0] = bf2_to_f2(r.w[0].x);
    o[1] = bf2_to_f2(r.w[0].y);
    o[2] = bf2_to_f2(r.w[0].z);
    o[3] = bf2_to_f2(r.w[0].w);
  }
}
__device__ __forceinline__ void gain8(const float* g, int64_t idx, float2 (&o)[4]) {
  if (!g) {
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = make_float2(1.0f, 1.0f);
    return;
  }
  const float4 a = __ldg(reinterpret_cast<const float4*>(g + idx));
  const float4 b = __ldg(reinterpret_cast<const float4*>(g + idx + 4));
  o[0] = make_float2(a.x, a.y); o[1] = make_float2(a.z, a.w);
  o[2] = make_float2(b.x, b.y); o[3] = make_float2(b.z, b.w);
}
__device__ __forceinline__ float2 silu2(float2 z) { return make_float2(siluf_(z.x), siluf_(z.y)); }

// Sum of squares of a thread's chunks: one packed accumulator per chunk, then a pairwise tree, so
// the dependent chains are four products long instead of 4 * NCH.
template <int NCH>
__device__ __forceinline__ float2 sumsq_tree(const float2 (&v)[NCH][4]) {
  float2 p[NCH];
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    p[i] = __fmul2_rn(v[i][0], v[i][0]);
#pragma unroll
    for (int e = 1; e < 4; ++e) p[i] = __ffma2_rn(v[i][e], v[i][e], p[i]);
  }
#pragma unroll
  for (int h = 1; h < NCH; h *= 2)
#pragma unroll
    for (int i = 0; i + h < NCH; i += 2 * h) p[i] = __fadd2_rn(p[i], p[i + h]);
  return p[0];
}

// Row group of W warps per row, NCH chunks of 8 values per thread (K <= 256 * W * NCH). The CTAs
// are persistent: each row group walks rows gridDim.x * (4 / W) apart. A thread sees the same
// columns in every row, so it holds their norm gains in registers for the whole launch, and it
// loads the next row's inputs into registers before it works on the current one, so a row's HBM
// latency overlaps the previous row's reductions and arithmetic. Element-wise products use packed
// f32x2 arithmetic (each lane rounds exactly as the scalar operation would).
template <mmf_dtype XT, int MODE, int W, int NCH, int NG>
__global__ void __launch_bounds__(kNqThreads) norm_quant_vec_kernel(const NormQuantArgs a) {
  constexpr int GT = 32 * W;
  constexpr int RPC = (kNqThreads / 32) / W;  // rows per CTA step
  constexpr bool TWO = MODE != kRowPlain;      // a second input: the up half (GLU) or g (g_norm)
  constexpr bool GN = MODE == kRowGnorm;
  __shared__ float reds[2][8];
  __shared__ float redm[2][8][3];
  int phs = 0, phm = 0;
  const int grp = (threadIdx.x >> 5) / W;
  const int gl = threadIdx.x - grp * GT;
  const int k = a.k, nck = k >> 3;
  const int64_t nrb = (a.m + RPC - 1) / RPC;
  Raw8<XT> rx[NCH], ry[TWO ? NCH : 1];
  float2 gr[NG][NCH][4], gwr[GN ? NCH : 1][4];
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = gl + i * GT;
#pragma unroll
    for (int j = 0; j < NG; ++j) {
      if (c < nck && j < a.ngain) gain8(a.gain[j], 8 * c, gr[j][i]);
      else
#pragma unroll
        for (int e = 0; e < 4; ++e) gr[j][i][e] = make_float2(0.0f, 0.0f);
    }
    if (GN) {
      if (c < nck) gain8(a.gw, 8 * c, gwr[GN ? i : 0]);
      else
#pragma unroll
        for (int e = 0; e < 4; ++e) gwr[GN ? i : 0][e] = make_float2(0.0f, 0.0f);
    }
  }

  auto fetch = [&](int64_t rb) {
    const int64_t row = rb * RPC + grp;
    if (rb < nrb && row < a.m) {
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        const int c = gl + i * GT;
        if (c < nck) {
          raw8_load<XT>(a.x, row * a.ldx + 8 * c, rx[i]);
          if (MODE == kRowGlu) raw8_load<XT>(a.x, row * a.ldx + k + 8 * c, ry[TWO ? i : 0]);
          if (MODE == kRowGnorm) raw8_load<XT>(a.g, row * a.ldg + 8 * c, ry[TWO ? i : 0]);
        }
      }
    }
  };

  int64_t rb = blockIdx.x;
  fetch(rb);
  for (; rb < nrb; rb += gridDim.x) {
    const int64_t row = rb * RPC + grp;
    const bool active = row < a.m;
    float2 v[NCH][4], y[TWO ? NCH : 1][4];
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = gl + i * GT;
      if (active && c < nck) {
        raw8_unpack<XT>(rx[i], v[i]);
        if (TWO) raw8_unpack<XT>(ry[TWO ? i : 0], y[TWO ? i : 0]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[i][e] = make_float2(0.0f, 0.0f);
          if (TWO) y[TWO ? i : 0][e] = make_float2(0.0f, 0.0f);
        }
      }
    }
    fetch(rb + gridDim.x);  // the next row's loads are in flight during the work below

    if (MODE == kRowGlu) {
#pragma unroll
      for (int i = 0; i < NCH; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) v[i][e] = __fmul2_rn(a.pre_act ? v[i][e] : silu2(v[i][e]), y[TWO ? i : 0][e]);
    }
    float2 ss2 = sumsq_tree<NCH>(v);
    if (GN) {
      // u = h / rms(h) * w_g * SiLU(g), then the BitLinear norm of u
      const float rfh = nq_rinv(nq_group_sum<W>(ss2.x + ss2.y, reds, phs), k, a.eps);
      const float2 rfh2 = make_float2(rfh, rfh);
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 sg = a.pre_act ? y[TWO ? i : 0][e] : silu2(y[TWO ? i : 0][e]);
          v[i][e] = __fmul2_rn(__fmul2_rn(__fmul2_rn(v[i][e], rfh2), gwr[GN ? i : 0][e]), sg);
        }
      }
      ss2 = sumsq_tree<NCH>(v);
    }
    const float rf = nq_rinv(nq_group_sum<W>(ss2.x + ss2.y, reds, phs), k, a.eps);
    const float2 rf2 = make_float2(rf, rf);
    // v <- v / rms (and, with one gain, <- r = v / rms * gain); maxima of |r| per gain
    float amax[NG];
    {
      float am[NG][NCH];  // per-chunk maxima, combined as a tree (max is exact in any order)
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        if (NG == 1) {
#pragma unroll
          for (int e = 0; e < 4; ++e) v[i][e] = __fmul2_rn(__fmul2_rn(v[i][e], rf2), gr[0][i][e]);
          am[0][i] = fmaxf(fmaxf(fabsf(v[i][0].x), fabsf(v[i][0].y)), fmaxf(fabsf(v[i][1].x), fabsf(v[i][1].y)));
          am[0][i] = fmaxf(am[0][i], fmaxf(fmaxf(fabsf(v[i][2].x), fabsf(v[i][2].y)), fmaxf(fabsf(v[i][3].x), fabsf(v[i][3].y))));
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) v[i][e] = __fmul2_rn(v[i][e], rf2);
#pragma unroll
          for (int j = 0; j < NG; ++j) {
            float2 r[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) r[e] = __fmul2_rn(v[i][e], gr[j][i][e]);
            am[j][i] = fmaxf(fmaxf(fmaxf(fabsf(r[0].x), fabsf(r[0].y)), fmaxf(fabsf(r[1].x), fabsf(r[1].y))),
                             fmaxf(fmaxf(fabsf(r[2].x), fabsf(r[2].y)), fmaxf(fabsf(r[3].x), fabsf(r[3].y))));
          }
        }
      }
#pragma unroll
      for (int j = 0; j < NG; ++j) {
#pragma unroll
        for (int h = 1; h < NCH; h *= 2)
#pragma unroll
          for (int i = 0; i + h < NCH; i += 2 * h) am[j][i] = fmaxf(am[j][i], am[j][i + h]);
        amax[j] = am[j][0];
      }
    }
    nq_group_max<W, NG>(amax, redm, phm);
    if (active) {
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        if (j < a.ngain) {
          const float am = fmaxf(amax[j], 1e-5f);
          const float sx = q127_over(am);
          const float2 sx2 = make_float2(sx, sx);
          int8_t* qrow = a.q[j] + row * a.ldq;
#pragma unroll
          for (int i = 0; i < NCH; ++i) {
            const int c = gl + i * GT;
            if (c < nck) {
              float2 b[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                b[e] = q8_add2(__fmul2_rn(NG == 1 ? v[i][e] : __fmul2_rn(v[i][e], gr[j][i][e]), sx2));
              *reinterpret_cast<uint2*>(qrow + 8 * c) = pack8_codes(b);
            }
          }
          for (int c = nck + gl; c < (int)(a.ldq >> 3); c += GT) *reinterpret_cast<uint2*>(qrow + 8 * c) = make_uint2(0u, 0u);
          if (gl == 0) a.deq[j][row] = over_127(am);
        }
      }
    }
  }
}

// =============================================================================================
// BitLinear segments (shared by both integer-product engines)
// =============================================================================================
struct GemmSeg {
  const int8_t* q;       // [m][ldq] activation codes (ldq = 16 * kw, padding columns are 0)
  const float* deq;      // [m] a/127 per row
  const uint32_t* codes; // [n][kw] packed weights
  const float* sw;       // weight scale (1 float)
  int32_t n;
  void* y;               // y[row * ldy + ycol + col]
  int64_t ldy;
  int32_t ycol;
  const void* res;       // optional residual, same dtype as y, res[row * ldres + rescol + col]
  int64_t ldres;
  int32_t rescol;
  int32_t* acc;          // optional raw accumulators acc[row * ldacc + col]
  int64_t ldacc;
  int32_t act;           // activation applied to output columns [0, act_cols): kActNone/Silu/SigmoidNeg
  int32_t act_cols;
  int32_t glu;           // 1: codes are [2 * glu_inner][kw] (gate rows, then up rows) and the output
  int32_t glu_inner;     //    is v[row][col] = SiLU(gate col) * up col, col < glu_inner (tensor engine)
};

struct GemmArgs {
  GemmSeg seg[3];
  int32_t nseg;
  int64_t m;
  int32_t k;
  int32_t kw;
  int64_t ldq;
  mmf_dtype ydt;
};

// Element-wise activations a BitLinear epilogue can apply to its output (the gates that follow
// the projections in the block, evaluated once where the value is produced).
enum ActKind : int32_t {
  kActNone = 0,
  kActSilu = 1,        // SiLU(z) = z * sigmoid(z)
  kActSigmoidNeg = 2   // sigmoid(-z) = 1 - sigmoid(z), the forget gate's complement
};
__device__ __forceinline__ float apply_act(int32_t act, float z) {
  if (act == kActSilu) return siluf_(z);
  if (act == kActSigmoidNeg) return __fdividef(1.0f, 1.0f + __expf(z));
  return z;
}

// y = act(acc * deq[row] * s (+ residual)), plus the optional raw accumulator.
__device__ __forceinline__ void bitlinear_epilogue(const GemmSeg& s, mmf_dtype ydt, int64_t row,
                                                   int32_t col, int32_t acc, float sw) {
  if (s.acc) s.acc[row * s.ldacc + col] = acc;
  float z = (float)acc * (s.deq[row] * sw);  // same rounding order as the tensor-core epilogue
  if (s.res) z += load_as_float(s.res, row * s.ldres + s.rescol + col, ydt);
  if (col < s.act_cols) z = apply_act(s.act, z);
  store_from_float(s.y, row * s.ldy + s.ycol + col, ydt, z);
}

// =============================================================================================
// K3: CUDA-core ternary GEMM for a few rows (decode) -- dp4a on expanded codes
// =============================================================================================
// Block = 8 warps; each warp owns 4 weight rows, 8 lanes per row; each lane streams 16-byte
// chunks (64 codes) of its row. The block's MT activation rows sit in shared memory arranged
// piece-major (piece p of chunk c at [p][c]) so the 8 lanes of a row read 128 contiguous bytes.
constexpr int kSimtMT = 8;

__global__ void __launch_bounds__(256) simt_gemm_kernel(const GemmArgs a) {
  extern __shared__ uint4 sact[];
  const GemmSeg& s = a.seg[blockIdx.z];
  const int64_t m0 = (int64_t)blockIdx.y * kSimtMT;
  const int mt = (int)(a.m - m0 < kSimtMT ? a.m - m0 : kSimtMT);
  const int nchunk = a.kw >> 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 3, l8 = lane & 7;
  // The first PF chunks of this lane's first weight row are loaded before the activations are
  // staged, so the weight stream is in flight while the block copies and synchronises.
  constexpr int PF = 8;
  uint4 wpf[PF];
  {
    const int n = blockIdx.x * 32 + warp * 4 + grp;
    const uint4* wrow = reinterpret_cast<const uint4*>(s.codes + (int64_t)(n < s.n ? n : 0) * a.kw);
#pragma unroll
    for (int p = 0; p < PF; ++p) {
      const int c = l8 + 8 * p;
      wpf[p] = (n < s.n && c < nchunk) ? __ldg(wrow + c) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  // stage activations
  for (int idx = threadIdx.x; idx < mt * nchunk * 4; idx += blockDim.x) {
    const int j = idx / (nchunk * 4);
    const int rem = idx - j * nchunk * 4;
    const int c = rem >> 2, p = rem & 3;
    sact[j * nchunk * 4 + p * nchunk + c] =
        *reinterpret_cast<const uint4*>(s.q + (m0 + j) * a.ldq + c * 64 + p * 16);
  }
  __syncthreads();
  const float sw = s.sw[0];
  bool first = true;
  for (int base = blockIdx.x * 32 + warp * 4; base < s.n; base += gridDim.x * 32) {
    const int n = base + grp;
    const bool valid = n < s.n;
    int acc[kSimtMT];
#pragma unroll
    for (int j = 0; j < kSimtMT; ++j) acc[j] = 0;
    const uint4* wrow = reinterpret_cast<const uint4*>(s.codes + (int64_t)(valid ? n : 0) * a.kw);
    auto consume = [&](const uint4& wv, int c) {
      uint32_t e[16];
      expand_word(wv.x, e + 0);
      expand_word(wv.y, e + 4);
      expand_word(wv.z, e + 8);
      expand_word(wv.w, e + 12);
#pragma unroll
      for (int j = 0; j < kSimtMT; ++j) {
        if (j < mt) {
          const uint4* arow = sact + j * nchunk * 4 + c;
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const uint4 av = arow[p * nchunk];
            acc[j] = __dp4a((int)e[4 * p + 0], (int)av.x, acc[j]);
            acc[j] = __dp4a((int)e[4 * p + 1], (int)av.y, acc[j]);
            acc[j] = __dp4a((int)e[4 * p + 2], (int)av.z, acc[j]);
            acc[j] = __dp4a((int)e[4 * p + 3], (int)av.w, acc[j]);
          }
        }
      }
    };
    int c0 = l8;
    if (first) {
#pragma unroll
      for (int p = 0; p < PF; ++p)
        if (l8 + 8 * p < nchunk) consume(wpf[p], l8 + 8 * p);
      c0 = l8 + 8 * PF;
      first = false;
    }
    for (int c = c0; c < nchunk; c += 8) {
      const uint4 wv = valid ? __ldg(wrow + c) : make_uint4(0u, 0u, 0u, 0u);
      consume(wv, c);
    }
#pragma unroll
    for (int j = 0; j < kSimtMT; ++j) {
      acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 4);
      acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 2);
      acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 1);
    }
    if (valid) {
#pragma unroll
      for (int j = 0; j < kSimtMT; ++j)
        if (j < mt && l8 == j) bitlinear_epilogue(s, a.ydt, m0 + j, n, acc[j], sw);
    }
  }
}

// =============================================================================================
// K4: HGRN scan with fused gates (chunked: aggregate -> carry -> replay)
// =============================================================================================
// The step h -> f h + i is affine, so a run of steps composes to h -> A h + B. The sequence is
// cut into chunks of `chunk` steps. Phase 1 folds every (channel, chunk) into its (A, B);
// phase 2 walks the chunks of each channel in order and records the state entering each chunk
// (and the final state); phase 3 replays every chunk from its entry state and stores h. Each
// thread owns VEC adjacent channels (paired 4- or 8-byte loads), lanes cover consecutive channel
// pairs, so every access is a coalesced row segment. Sequences no longer than one chunk (decode)
// take the single-pass kernel instead.
struct ScanArgs {
  const void* zf;
  const void* zi;
  mmf_dtype zdt;
  int64_t zstride;  // elements between consecutive time steps (row stride)
  int32_t b;
  int64_t t;
  int32_t d;
  const float* h0;
  void* h;          // [b][t][d]
  mmf_dtype hdt;
  float* h_last;
  int32_t chunk;    // steps per chunk
  int32_t nchunk;
  float* agg_a;     // [b][nchunk][d]
  float* agg_b;     // [b][nchunk][d]
  float* cin;       // [b][nchunk][d] state entering each chunk
  int32_t gated;    // 0: zf, zi are gate pre-activations; 1: zf holds 1 - f, zi holds SiLU(zi)
};
constexpr int kScanThreads = 128;

template <mmf_dtype DT, int VEC>
__device__ __forceinline__ void load_vec(const void* base, int64_t idx, float (&o)[VEC]) {
  if (VEC == 2) {
    if (DT == MMF_F32) {
      const float2 v = *reinterpret_cast<const float2*>(reinterpret_cast<const float*>(base) + idx);
      o[0] = v.x;
      o[VEC - 1] = v.y;
    } else {
      const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(
          reinterpret_cast<const __nv_bfloat16*>(base) + idx));
      o[0] = v.x;
      o[VEC - 1] = v.y;
    }
  } else {
    o[0] = Elem<DT>::load(reinterpret_cast<const typename Elem<DT>::T*>(base) + idx);
  }
}
template <mmf_dtype DT, int VEC>
__device__ __forceinline__ void store_vec(void* base, int64_t idx, const float (&v)[VEC]) {
  if (VEC == 2) {
    if (DT == MMF_F32)
      *reinterpret_cast<float2*>(reinterpret_cast<float*>(base) + idx) = make_float2(v[0], v[VEC - 1]);
    else
      *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(base) + idx) =
          __floats2bfloat162_rn(v[0], v[VEC - 1]);
  } else {
    Elem<DT>::store(reinterpret_cast<typename Elem<DT>::T*>(base) + idx, v[0]);
  }
}

// f = sigmoid(zf), i = SiLU(zi) * (1 - f); with GATED the inputs already are (1 - f, SiLU(zi)).
template <bool GATED>
__device__ __forceinline__ void hgrn_gate(float zf, float zi, float& f, float& i) {
  if (GATED) {
    f = 1.0f - zf;
    i = zi * zf;
  } else {
    float omf;
    hgrn_forget(zf, f, omf);
    i = siluf_(zi) * omf;
  }
}

// The gates of two channels with packed f32x2 arithmetic and one reciprocal per channel: with
// ef = e^-zf and ez = e^-zi, f = 1/(1+ef), 1 - f = ef/(1+ef) and sigmoid(zi) = 1/(1+ez), so
// r = 1/((1+ef)(1+ez)) gives f = (1+ez) r and i = SiLU(zi)(1 - f) = zi ef r: three MUFU
// operations per channel instead of four, no cancellation in 1 - f. Both exponent arguments are
// clamped at -40 so the product stays finite (below 2^116, no inf * 0); sigmoid(-40) < 5e-18, so
// the clamp moves f or i by less than 5e-18 |zi|. With GATED the inputs already are
// (1 - f, SiLU(zi)).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
template <bool GATED>
__device__ __forceinline__ void hgrn_gate2(float2 zf, float2 zi, float2& f, float2& i) {
  const float2 one = make_float2(1.0f, 1.0f);
  if (GATED) {
    f = __fadd2_rn(one, make_float2(-zf.x, -zf.y));
    i = __fmul2_rn(zi, zf);
  } else {
    constexpr float kNegLog2e = -1.4426950408889634f;
    const float2 nl = make_float2(kNegLog2e, kNegLog2e);
    const float2 xf = __fmul2_rn(make_float2(fmaxf(zf.x, -40.0f), fmaxf(zf.y, -40.0f)), nl);
    const float2 xi = __fmul2_rn(make_float2(fmaxf(zi.x, -40.0f), fmaxf(zi.y, -40.0f)), nl);
    const float2 ef = make_float2(ex2_approx(xf.x), ex2_approx(xf.y));
    const float2 ez = make_float2(ex2_approx(xi.x), ex2_approx(xi.y));
    const float2 pz = __fadd2_rn(ez, one);
    const float2 den = __fmul2_rn(__fadd2_rn(ef, one), pz);
    const float2 r = make_float2(rcp_approx(den.x), rcp_approx(den.y));
    f = __fmul2_rn(pz, r);
    i = __fmul2_rn(__fmul2_rn(zi, ef), r);
  }
}

// Steps loaded ahead into registers before the dependent recurrence runs over them.
constexpr int kScanPrefetch = 16;  // = the chunk length for sequences up to 2048 steps

template <mmf_dtype ZT, int VEC>
__device__ __forceinline__ void scan_load_block(const ScanArgs& a, int64_t zb, int64_t t, int64_t t1,
                                                float (&zf)[kScanPrefetch][VEC], float (&zi)[kScanPrefetch][VEC]) {
#pragma unroll
  for (int u = 0; u < kScanPrefetch; ++u) {
    if (t + u < t1) {
      load_vec<ZT, VEC>(a.zf, zb + (t + u) * a.zstride, zf[u]);
      load_vec<ZT, VEC>(a.zi, zb + (t + u) * a.zstride, zi[u]);
    }
  }
}

template <mmf_dtype ZT, int VEC, bool GATED>
__global__ void __launch_bounds__(kScanThreads) scan_aggregate_kernel(const ScanArgs a) {
  const int64_t ch = ((int64_t)blockIdx.x * kScanThreads + threadIdx.x) * VEC;
  if (ch >= a.d) return;
  const int c = blockIdx.y, bi = blockIdx.z;
  const int64_t t0 = (int64_t)c * a.chunk;
  const int64_t t1 = t0 + a.chunk < a.t ? t0 + a.chunk : a.t;
  const int64_t zb = (int64_t)bi * a.t * a.zstride + ch;
  float A[VEC], B[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) { A[v] = 1.0f; B[v] = 0.0f; }
  for (int64_t t = t0; t < t1; t += kScanPrefetch) {
    float zf[kScanPrefetch][VEC], zi[kScanPrefetch][VEC];
    scan_load_block<ZT, VEC>(a, zb, t, t1, zf, zi);
#pragma unroll
    for (int u = 0; u < kScanPrefetch; ++u) {
      if (t + u < t1) {
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
          float f, i;
          hgrn_gate<GATED>(zf[u][v], zi[u][v], f, i);
          A[v] = f * A[v];
          B[v] = f * B[v] + i;
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

__global__ void __launch_bounds__(kScanThreads) scan_carry_kernel(const ScanArgs a) {
  const int64_t ch = (int64_t)blockIdx.x * kScanThreads + threadIdx.x;
  if (ch >= a.d) return;
  const int bi = blockIdx.y;
  const float* __restrict__ A = a.agg_a;
  const float* __restrict__ B = a.agg_b;
  float* __restrict__ cin = a.cin;
  float carry = a.h0 ? a.h0[(int64_t)bi * a.d + ch] : 0.0f;
  const int64_t base = (int64_t)bi * a.nchunk * a.d + ch;
  constexpr int PF = 32;
  for (int c0 = 0; c0 < a.nchunk; c0 += PF) {
    float av[PF], bv[PF];
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      if (c0 + u < a.nchunk) {
        av[u] = A[base + (int64_t)(c0 + u) * a.d];
        bv[u] = B[base + (int64_t)(c0 + u) * a.d];
      }
    }
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      if (c0 + u < a.nchunk) {
        cin[base + (int64_t)(c0 + u) * a.d] = carry;
        carry = av[u] * carry + bv[u];
      }
    }
  }
  if (a.h_last) a.h_last[(int64_t)bi * a.d + ch] = carry;
}

// Replays chunk c from its entry state (phase 3); with SINGLE the whole sequence is one chunk
// entered from h0 and the final state is written too.
template <mmf_dtype ZT, mmf_dtype HT, int VEC, bool SINGLE, bool GATED>
__global__ void __launch_bounds__(kScanThreads) scan_apply_kernel(const ScanArgs a) {
  const int64_t ch = ((int64_t)blockIdx.x * kScanThreads + threadIdx.x) * VEC;
  if (ch >= a.d) return;
  const int c = blockIdx.y, bi = blockIdx.z;
  const int64_t t0 = (int64_t)c * a.chunk;
  const int64_t t1 = t0 + a.chunk < a.t ? t0 + a.chunk : a.t;
  const int64_t zb = (int64_t)bi * a.t * a.zstride + ch;
  const int64_t hb = (int64_t)bi * a.t * a.d + ch;
  float h[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) {
    if (SINGLE) h[v] = a.h0 ? a.h0[(int64_t)bi * a.d + ch + v] : 0.0f;
    else h[v] = a.cin[((int64_t)bi * a.nchunk + c) * a.d + ch + v];
  }
  for (int64_t t = t0; t < t1; t += kScanPrefetch) {
    float zf[kScanPrefetch][VEC], zi[kScanPrefetch][VEC];
    scan_load_block<ZT, VEC>(a, zb, t, t1, zf, zi);
#pragma unroll
    for (int u = 0; u < kScanPrefetch; ++u) {
      if (t + u < t1) {
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
          float f, i;
          hgrn_gate<GATED>(zf[u][v], zi[u][v], f, i);
          h[v] = f * h[v] + i;
        }
        store_vec<HT, VEC>(a.h, hb + (t + u) * a.d, h);
      }
    }
  }
  if (SINGLE && a.h_last) {
#pragma unroll
    for (int v = 0; v < VEC; ++v) a.h_last[(int64_t)bi * a.d + ch + v] = h[v];
  }
}

// Tiled variant of the aggregate / apply / single-pass phases for 16-byte aligned rows: a CTA of
// kScanThreads threads owns kScanTileCh channels (two per thread) and streams its chunk through
// shared memory in tiles of kScanTileSteps steps with double-buffered cp.async copies, so many
// KB per SM are in flight without holding them in registers. Chunks are 64 steps (four tiles),
// and the gates of a channel pair are formed with packed f32x2 arithmetic (hgrn_gate2): both
// phases are bound by the MUFU and issue rates, not by HBM. (A single-pass variant chaining the
// chunks by decoupled look-back, which reads z once, measured slower on B200: the per-chunk
// publish / poll latency outweighed the second read.)
constexpr int kScanTileCh = 2 * kScanThreads;  // 256 channels per CTA
constexpr int kScanTileSteps = 16;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <mmf_dtype ZT>
constexpr int scan_tile_bytes() {
  return 2 /*stages*/ * 2 /*zf, zi*/ * kScanTileSteps * kScanTileCh * (ZT == MMF_F32 ? 4 : 2);
}

// PHASE 0: aggregates; 1: replay from the chunk's entry state; 2: single chunk from h0 (+ h_last).
template <mmf_dtype ZT, mmf_dtype HT, bool GATED, int PHASE>
__global__ void __launch_bounds__(kScanThreads) scan_tile_kernel(const ScanArgs a) {
  constexpr int ES = ZT == MMF_F32 ? 4 : 2;
  constexpr int ROWB = kScanTileCh * ES;                    // bytes of one step row of one array
  constexpr int PIECES = 2 * kScanTileSteps * ROWB / 16;    // 16-byte copies per stage
  extern __shared__ __align__(16) uint8_t scan_sm[];
  const int tid = threadIdx.x;
  const int64_t ch0 = (int64_t)blockIdx.x * kScanTileCh;
  const int c = blockIdx.y, bi = blockIdx.z;
  const int64_t t0 = (int64_t)c * a.chunk;
  const int64_t t1 = t0 + a.chunk < a.t ? t0 + a.chunk : a.t;
  const int nblk = (int)((t1 - t0 + kScanTileSteps - 1) / kScanTileSteps);
  const int64_t row_bytes_valid = (a.d - ch0) * ES < ROWB ? (a.d - ch0) * ES : ROWB;
  const uint8_t* zfb = reinterpret_cast<const uint8_t*>(a.zf);
  const uint8_t* zib = reinterpret_cast<const uint8_t*>(a.zi);

  auto issue = [&](int stage, int blk) {
    uint8_t* dst0 = scan_sm + stage * (2 * kScanTileSteps * ROWB);
    for (int p = tid; p < PIECES; p += kScanThreads) {
      const int arr = p / (PIECES / 2);
      const int rem = p - arr * (PIECES / 2);
      const int u = rem / (ROWB / 16), col = (rem - u * (ROWB / 16)) * 16;
      const int64_t t = t0 + (int64_t)blk * kScanTileSteps + u;
      if (t < t1 && col < row_bytes_valid) {
        const uint8_t* src = (arr ? zib : zfb) + (((int64_t)bi * a.t + t) * a.zstride + ch0) * ES + col;
        cp_async16(dst0 + (arr * kScanTileSteps + u) * ROWB + col, src);
      }
    }
    cp_async_commit();
  };

  const int64_t ch = ch0 + 2 * tid;
  const bool valid = ch < a.d;  // d is even on this path
  float2 Av = make_float2(1.0f, 1.0f), Bv = make_float2(0.0f, 0.0f), hv = make_float2(0.0f, 0.0f);
  if (valid) {
    if (PHASE == 1) hv = *reinterpret_cast<const float2*>(a.cin + ((int64_t)bi * a.nchunk + c) * a.d + ch);
    else if (PHASE == 2 && a.h0) hv = *reinterpret_cast<const float2*>(a.h0 + (int64_t)bi * a.d + ch);
  }
  issue(0, 0);
  for (int blk = 0; blk < nblk; ++blk) {
    if (blk + 1 < nblk) {
      issue((blk + 1) & 1, blk + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint8_t* st = scan_sm + (blk & 1) * (2 * kScanTileSteps * ROWB);
    const int64_t tb = t0 + (int64_t)blk * kScanTileSteps;
    const int steps = t1 - tb < kScanTileSteps ? (int)(t1 - tb) : kScanTileSteps;
    auto step = [&](int u) {
      float zf[2], zi[2];
      load_vec<ZT, 2>(st + (0 * kScanTileSteps + u) * ROWB, 2 * tid, zf);
      load_vec<ZT, 2>(st + (1 * kScanTileSteps + u) * ROWB, 2 * tid, zi);
      float2 f, i;
      hgrn_gate2<GATED>(make_float2(zf[0], zf[1]), make_float2(zi[0], zi[1]), f, i);
      if (PHASE == 0) {
        Av = __fmul2_rn(Av, f);
        Bv = __ffma2_rn(f, Bv, i);
      } else {
        hv = __ffma2_rn(f, hv, i);
        const float o[2] = {hv.x, hv.y};
        store_vec<HT, 2>(a.h, ((int64_t)bi * a.t + tb + u) * a.d + ch, o);
      }
    };
    if (valid) {
      if (steps == kScanTileSteps) {
#pragma unroll
        for (int u = 0; u < kScanTileSteps; ++u) step(u);
      } else {
        for (int u = 0; u < steps; ++u) step(u);
      }
    }
    __syncthreads();  // the stage is refilled by the next iteration's copies
  }
  if (!valid) return;
  if (PHASE == 0) {
    const int64_t o = ((int64_t)bi * a.nchunk + c) * a.d + ch;
    *reinterpret_cast<float2*>(a.agg_a + o) = Av;
    *reinterpret_cast<float2*>(a.agg_b + o) = Bv;
  } else if (PHASE == 2 && a.h_last) {
    *reinterpret_cast<float2*>(a.h_last + (int64_t)bi * a.d + ch) = hv;
  }
}

// =============================================================================================
// K7: embedding gather
// =============================================================================================
__global__ void __launch_bounds__(256) embed_gather_kernel(const int32_t* __restrict__ ids, int64_t m,
                                                           const void* __restrict__ table,
                                                           mmf_dtype dt, int32_t vocab, int32_t d,
                                                           void* __restrict__ out) {
  const int64_t row = blockIdx.x;
  if (row >= m) return;
  const int32_t id = ids[row];
  const bool ok = id >= 0 && id < vocab;
  const int es = dt == MMF_F32 ? 4 : 2;
  const int64_t bytes = (int64_t)d * es;
  const uint8_t* src = reinterpret_cast<const uint8_t*>(table) + (ok ? (int64_t)id * bytes : 0);
  uint8_t* dst = reinterpret_cast<uint8_t*>(out) + row * bytes;
  if ((bytes & 15) == 0) {
    for (int64_t i = threadIdx.x; i < bytes / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(dst)[i] = ok ? reinterpret_cast<const uint4*>(src)[i] : make_uint4(0, 0, 0, 0);
  } else {
    for (int64_t i = threadIdx.x; i < bytes; i += blockDim.x) dst[i] = ok ? src[i] : 0;
  }
}

// Debug taps: dst[r][c] = float(src[r][c]) for r < rows, c < cols (row strides in elements).
__global__ void __launch_bounds__(256) tap_to_f32_kernel(const void* __restrict__ src, mmf_dtype sdt, int64_t rows,
                                                         int32_t cols, int64_t src_ld, float* __restrict__ dst,
                                                         int64_t dst_ld) {
  const int64_t total = rows * cols;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / cols, c = e - r * cols;
    dst[r * dst_ld + c] = load_as_float(src, r * src_ld + c, sdt);
  }
}

}  // namespace mmf
