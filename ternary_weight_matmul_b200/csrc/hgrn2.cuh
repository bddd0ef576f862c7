// hgrn2.cuh -- HGRN2 recurrence with state expansion, step by step on the CUDA cores.
//
//   S_t = diag(f_t) S_{t-1} + (1 - f_t)^T i_t      (S: dk x dv per sequence and head)
//   o_t = q_t S_t
//
// HGRN2 is named by the MatMul-Free LLM report (nightvoyager.top, innovations table: gated
// linear recurrence with fused-recurrent and chunked kernels); the recurrence is HGRN2's
// published one. Column v of the state sees only i_t[v], so the dv columns evolve independently:
// one thread owns one column, keeps its dk state values in registers for the whole sequence and
// forms o_t[v] as the dot product of q_t with them, with no exchange between threads. A CTA
// serves 128 columns of one (sequence, head); per tile of kTS steps it stages q_t and f_t (dk
// values each, shared by every column) in shared memory as float32. Rows past dk are padded with
// q = 0 and f = 1 (key 0), so they stay zero and never contribute.
#pragma once

#include "common.cuh"

namespace mmf {
namespace hgrn2 {

constexpr int kThreads = 128;   // value columns per CTA
constexpr int kTS = 16;         // steps per staged tile

struct Args {
  const void* q;       // [b][t][heads][dk]
  const void* f;       // [b][t][heads][dk], forget gates in [0, 1]
  const void* i;       // [b][t][heads][dv]
  mmf_dtype dt;        // of q, f, i and o
  int32_t b;
  int64_t t;
  int32_t heads;
  int32_t dk;          // <= DK of the instance
  int32_t dv;
  const float* s0;     // [b][heads][dk][dv] or null (zeros)
  float* s_out;        // [b][heads][dk][dv] or null
  void* o;             // [b][t][heads][dv]
};

template <mmf_dtype DT, int DK>
__global__ void __launch_bounds__(kThreads) hgrn2_recurrent_kernel(const Args a) {
  using T = typename Elem<DT>::T;
  __shared__ __align__(16) float qs[kTS][DK];
  __shared__ __align__(16) float fs[kTS][DK];
  const int v = blockIdx.x * kThreads + threadIdx.x;
  const int h = blockIdx.y, bi = blockIdx.z;
  const bool active = v < a.dv;
  const int64_t qk_step = (int64_t)a.heads * a.dk;   // elements of q / f per step
  const int64_t iv_step = (int64_t)a.heads * a.dv;   // elements of i / o per step
  const T* q = reinterpret_cast<const T*>(a.q) + (int64_t)bi * a.t * qk_step + (int64_t)h * a.dk;
  const T* f = reinterpret_cast<const T*>(a.f) + (int64_t)bi * a.t * qk_step + (int64_t)h * a.dk;
  const T* in = reinterpret_cast<const T*>(a.i) + (int64_t)bi * a.t * iv_step + (int64_t)h * a.dv;
  T* o = reinterpret_cast<T*>(a.o) + (int64_t)bi * a.t * iv_step + (int64_t)h * a.dv;
  const int64_t s_base = ((int64_t)bi * a.heads + h) * a.dk * a.dv;

  float S[DK];
#pragma unroll
  for (int k = 0; k < DK; ++k) S[k] = (a.s0 && active && k < a.dk) ? a.s0[s_base + (int64_t)k * a.dv + v] : 0.0f;

  for (int64_t t0 = 0; t0 < a.t; t0 += kTS) {
    const int ns = (int)(a.t - t0 < kTS ? a.t - t0 : kTS);
    __syncthreads();  // every column is done with the previous tile
    for (int e = threadIdx.x; e < kTS * DK; e += kThreads) {
      const int s = e / DK, k = e - s * DK;
      float qv = 0.0f, fv = 1.0f;
      if (s < ns && k < a.dk) {
        qv = Elem<DT>::load(q + (t0 + s) * qk_step + k);
        fv = Elem<DT>::load(f + (t0 + s) * qk_step + k);
      }
      qs[s][k] = qv;
      fs[s][k] = fv;
    }
    __syncthreads();
    if (active) {
      for (int s = 0; s < ns; ++s) {
        const float iv = Elem<DT>::load(in + (t0 + s) * iv_step + v);
        float acc = 0.0f;
#pragma unroll
        for (int k = 0; k < DK; k += 4) {
          const float4 f4 = *reinterpret_cast<const float4*>(&fs[s][k]);
          const float4 q4 = *reinterpret_cast<const float4*>(&qs[s][k]);
          S[k] = fmaf(f4.x, S[k], (1.0f - f4.x) * iv);
          S[k + 1] = fmaf(f4.y, S[k + 1], (1.0f - f4.y) * iv);
          S[k + 2] = fmaf(f4.z, S[k + 2], (1.0f - f4.z) * iv);
          S[k + 3] = fmaf(f4.w, S[k + 3], (1.0f - f4.w) * iv);
          acc = fmaf(q4.x, S[k], acc);
          acc = fmaf(q4.y, S[k + 1], acc);
          acc = fmaf(q4.z, S[k + 2], acc);
          acc = fmaf(q4.w, S[k + 3], acc);
        }
        Elem<DT>::store(o + (t0 + s) * iv_step + v, acc);
      }
    }
  }
  if (active && a.s_out) {
#pragma unroll
    for (int k = 0; k < DK; ++k)
      if (k < a.dk) a.s_out[s_base + (int64_t)k * a.dv + v] = S[k];
  }
}

}  // namespace hgrn2
}  // namespace mmf
