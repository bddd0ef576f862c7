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
// One thread per (sequence, channel) walks the steps in reverse, reading zf, zi, dh and the
// forward's h_{t-1} and writing dzf, dzi: consecutive threads take consecutive channels, so every
// access is coalesced across the warp. f_{t+1} is carried in a register from the previous
// (later) step.
//
// FusedBitLinear with the straight-through estimator (the report: weight_quant quantises in the
// forward pass and keeps the gradient in the backward pass; the activation quantiser is taken the
// same way): with the forward's codes q and factors a/127, the dequantised operands are
// rq = q (a/127) and Wq = t s, and
//   dr = dy Wq;  u = dr w;  rho = (mean(x^2) + eps)^(-1/2);  dx = rho u - rho^3 x mean(u x);
//   dw[k] = sum_m dr[m][k] x[m][k] rho_m;  dW = dy^T rq  (the latent weight's gradient).
// Five small CUDA-core kernels, in this order: rho per row; dr per (row, 16-column word of the
// packed codes), written into dx's buffer; the gain's gradient per column; dx per row, in place
// over dr; dW per (weight row, column).
#pragma once

#include "common.cuh"

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
};

template <mmf_dtype DT>
__global__ void __launch_bounds__(kThreads) scan_bwd_kernel(const ScanBwdArgs a) {
  using T = typename Elem<DT>::T;
  const int64_t gid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (gid >= (int64_t)a.b * a.d) return;
  const int bi = (int)(gid / a.d), c = (int)(gid - (int64_t)bi * a.d);
  const int64_t base = (int64_t)bi * a.t * a.d + c;
  const T* zf = reinterpret_cast<const T*>(a.zf);
  const T* zi = reinterpret_cast<const T*>(a.zi);
  const T* h = reinterpret_cast<const T*>(a.h);
  const T* dh = reinterpret_cast<const T*>(a.dh);
  T* dzf = reinterpret_cast<T*>(a.dzf);
  T* dzi = reinterpret_cast<T*>(a.dzi);
  const float h_init = a.h0 ? a.h0[(int64_t)bi * a.d + c] : 0.0f;
  float G = 0.0f, f_next = 0.0f;
  for (int64_t s = a.t - 1; s >= 0; --s) {
    const int64_t idx = base + s * a.d;
    G = fmaf(f_next, G, Elem<DT>::load(dh + idx));
    const float hp = s > 0 ? Elem<DT>::load(h + idx - a.d) : h_init;
    float f, omf;
    hgrn_forget(Elem<DT>::load(zf + idx), f, omf);
    const float z = Elem<DT>::load(zi + idx);
    const float sz = sigmoidf_(z);
    const float df = G * hp;
    Elem<DT>::store(dzf + idx, (df - G * (z * sz)) * f * omf);
    Elem<DT>::store(dzi + idx, G * omf * sz * fmaf(z, 1.0f - sz, 1.0f));
    f_next = f;
  }
  if (a.dh0) a.dh0[(int64_t)bi * a.d + c] = f_next * G;
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

// rho_m = (mean(x_m^2) + eps)^(-1/2), one warp per row.
__global__ void __launch_bounds__(kThreads) lin_bwd_rho_kernel(const LinBwdArgs a) {
  const int64_t row = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.m) return;
  float ss = 0.0f;
  for (int c = lane; c < a.k; c += 32) {
    const float v = load_as_float(a.x, row * a.k + c, a.xdt);
    ss = fmaf(v, v, ss);
  }
  ss = warp_sum(ss);
  if (lane == 0) a.rho[row] = rsqrtf(ss / (float)a.k + a.eps);
}

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

// dw[c] = sum_m dr[m][c] x[m][c] rho_m, one thread per column (coalesced across columns); m = 0
// gives zeros.
__global__ void __launch_bounds__(kThreads) lin_bwd_dnw_kernel(const LinBwdArgs a) {
  const int c = blockIdx.x * kThreads + threadIdx.x;
  if (c >= a.k) return;
  float acc = 0.0f;
  for (int64_t row = 0; row < a.m; ++row)
    acc = fmaf(a.dx[row * a.k + c] * load_as_float(a.x, row * a.k + c, a.xdt), a.rho[row], acc);
  a.dnorm_w[c] = acc;
}

// dx = rho u - rho^3 x mean(u x) with u = dr w, one CTA per row, in place over dr.
__global__ void __launch_bounds__(kThreads) lin_bwd_dx_kernel(const LinBwdArgs a) {
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  float* d = a.dx + row * a.k;
  float ux = 0.0f;
  for (int c = threadIdx.x; c < a.k; c += kThreads) {
    const float u = d[c] * (a.norm_w ? a.norm_w[c] : 1.0f);
    ux = fmaf(u, load_as_float(a.x, row * a.k + c, a.xdt), ux);
  }
  const float mean_ux = block_sum(ux, red) / (float)a.k;
  const float r = a.rho[row];
  const float r3 = r * r * r;
  for (int c = threadIdx.x; c < a.k; c += kThreads) {
    const float u = d[c] * (a.norm_w ? a.norm_w[c] : 1.0f);
    d[c] = r * u - r3 * load_as_float(a.x, row * a.k + c, a.xdt) * mean_ux;
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

}  // namespace bwd
}  // namespace mmf
