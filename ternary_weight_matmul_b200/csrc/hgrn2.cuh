// hgrn2.cuh -- HGRN2 recurrence with state expansion, step by step on the CUDA cores.
//
//   S_t = diag(f_t) S_{t-1} + (1 - f_t)^T i_t      (S: dk x dv per sequence and head)
//   o_t = q_t S_t
//
// HGRN2 is named by the MatMul-Free LLM report (nightvoyager.top, innovations table: gated
// linear recurrence with fused-recurrent and chunked kernels); the recurrence is HGRN2's
// published one. Column v of the state sees only i_t[v], so the dv columns evolve independently,
// and within a column every state row k evolves on its own (S[k][v] = f[k] S[k][v] + (1 - f[k])
// i[v]); only the readout o_t[v] = q_t . S_t[:, v] sums over k. Four adjacent threads share one
// column, each keeping dk / 4 state rows in registers for the whole sequence, and combine their
// partial readouts with two shuffles per step; the partial readout runs as four independent FMA
// chains. Thread `sub` of a column owns the rows 16 g + 4 sub + (0..3) for g = 0, 1, ..., so the
// four threads' 16-byte reads of q_t and f_t at one g are adjacent (no bank conflict). A CTA serves 32 columns of one (sequence, head); per tile of kTS steps it stages q_t and
// f_t (dk values each, shared by every column) in shared memory as float32. Rows past dk are
// padded with q = 0 and f = 1 (key 0), so they stay zero and never contribute.
#pragma once

#include "common.cuh"

namespace mmf {
namespace hgrn2 {

constexpr int kThreads = 128;   // threads per CTA
constexpr int kSplit = 4;       // threads per value column (each owns dk / kSplit state rows)
constexpr int kCols = kThreads / kSplit;  // value columns per CTA
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
  constexpr int KR = DK / kSplit;  // state rows per thread
  __shared__ __align__(16) float qs[kTS][DK];
  __shared__ __align__(16) float fs[kTS][DK];
  const int sub = threadIdx.x & (kSplit - 1);
  // state row of register j: 16 (j / 4) + 4 sub + j % 4
  auto krow = [&](int j) { return 16 * (j >> 2) + 4 * sub + (j & 3); };
  const int v = blockIdx.x * kCols + (threadIdx.x >> 2);
  const int h = blockIdx.y, bi = blockIdx.z;
  const bool active = v < a.dv;
  const int64_t qk_step = (int64_t)a.heads * a.dk;   // elements of q / f per step
  const int64_t iv_step = (int64_t)a.heads * a.dv;   // elements of i / o per step
  const T* q = reinterpret_cast<const T*>(a.q) + (int64_t)bi * a.t * qk_step + (int64_t)h * a.dk;
  const T* f = reinterpret_cast<const T*>(a.f) + (int64_t)bi * a.t * qk_step + (int64_t)h * a.dk;
  const T* in = reinterpret_cast<const T*>(a.i) + (int64_t)bi * a.t * iv_step + (int64_t)h * a.dv;
  T* o = reinterpret_cast<T*>(a.o) + (int64_t)bi * a.t * iv_step + (int64_t)h * a.dv;
  const int64_t s_base = ((int64_t)bi * a.heads + h) * a.dk * a.dv;

  float S[KR];
#pragma unroll
  for (int j = 0; j < KR; ++j)
    S[j] = (a.s0 && active && krow(j) < a.dk) ? a.s0[s_base + (int64_t)krow(j) * a.dv + v] : 0.0f;

  // The next tile's q, f (kTS x DK values spread over the CTA) and this column's i (kTS values)
  // are loaded into registers while the current tile runs, so no step waits on global memory.
  constexpr int PER = kTS * DK / kThreads;
  static_assert(PER * kThreads == kTS * DK, "tile split");
  T rq[PER], rf[PER], ri[kTS];
  auto load_tile = [&](int64_t tt) {
    const int nn = (int)(a.t - tt < kTS ? a.t - tt : kTS);
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int e = threadIdx.x + r * kThreads;
      const int st = e / DK, k = e - st * DK;
      if (st < nn && k < a.dk) {
        rq[r] = q[(tt + st) * qk_step + k];
        rf[r] = f[(tt + st) * qk_step + k];
      }
    }
#pragma unroll
    for (int st = 0; st < kTS; ++st)
      if (active && st < nn) ri[st] = in[(tt + st) * iv_step + v];
  };
  if (a.t > 0) load_tile(0);
  for (int64_t t0 = 0; t0 < a.t; t0 += kTS) {
    const int ns = (int)(a.t - t0 < kTS ? a.t - t0 : kTS);
    __syncthreads();  // every column is done with the previous tile
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int e = threadIdx.x + r * kThreads;
      const int st = e / DK, k = e - st * DK;
      const bool live = st < ns && k < a.dk;
      qs[st][k] = live ? Elem<DT>::to_float(rq[r]) : 0.0f;
      fs[st][k] = live ? Elem<DT>::to_float(rf[r]) : 1.0f;
    }
    float ivs[kTS];
#pragma unroll
    for (int st = 0; st < kTS; ++st) ivs[st] = active && st < ns ? Elem<DT>::to_float(ri[st]) : 0.0f;
    __syncthreads();
    if (t0 + kTS < a.t) load_tile(t0 + kTS);
    // (inactive columns take part in the shuffles with zero contributions)
#pragma unroll 1
    for (int s = 0; s < ns; ++s) {
      float iv = ivs[0];
#pragma unroll
      for (int st = 1; st < kTS; ++st) iv = s == st ? ivs[st] : iv;
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < KR; j += 4) {
        const float4 f4 = *reinterpret_cast<const float4*>(&fs[s][krow(j)]);
        const float4 q4 = *reinterpret_cast<const float4*>(&qs[s][krow(j)]);
        S[j] = fmaf(f4.x, S[j], (1.0f - f4.x) * iv);
        S[j + 1] = fmaf(f4.y, S[j + 1], (1.0f - f4.y) * iv);
        S[j + 2] = fmaf(f4.z, S[j + 2], (1.0f - f4.z) * iv);
        S[j + 3] = fmaf(f4.w, S[j + 3], (1.0f - f4.w) * iv);
        acc[0] = fmaf(q4.x, S[j], acc[0]);
        acc[1] = fmaf(q4.y, S[j + 1], acc[1]);
        acc[2] = fmaf(q4.z, S[j + 2], acc[2]);
        acc[3] = fmaf(q4.w, S[j + 3], acc[3]);
      }
      float part = (acc[0] + acc[1]) + (acc[2] + acc[3]);
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      if (active && sub == 0) Elem<DT>::store(o + (t0 + s) * iv_step + v, part);
    }
  }
  if (active && a.s_out) {
#pragma unroll
    for (int j = 0; j < KR; ++j)
      if (krow(j) < a.dk) a.s_out[s_base + (int64_t)krow(j) * a.dv + v] = S[j];
  }
}

}  // namespace hgrn2
}  // namespace mmf
