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

}  // namespace bwd
}  // namespace mmf
