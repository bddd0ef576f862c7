// decode_rows.cuh -- the row stages of a decode step on the skinny tensor-core path.
//
// A decode step of B <= 64 token rows runs each projection group as one skinny tensor-core
// product (gemm_skinny.cuh: the exact int32 accumulators acc[row][channel]) followed by one row
// stage here, which applies that group's epilogue and quantises the vector the next group
// consumes:
//   kQuantIn  x -> codes of x with the three i / f / g norm gains (the step's first layer);
//   kIFG      z = acc * (a/127) * s for i, f, g; f = sigmoid(zf), i = SiLU(zi) (1 - f),
//             h = f * h_prev + i (the carried state, updated in place);
//             u = RMSNorm(h) * gnorm_w * SiLU(g); codes of u with o_proj's gain;
//   kO        x1 = x + o (rounded to the activation dtype); codes of x1 with gate_proj's gain;
//   kGate     v = SiLU(gate) * up (rounded to the activation dtype); codes of v with down_proj's
//             gain;
//   kDown     y = x1 + down (rounded); codes of y with the next layer's three gains, if any.
// One CTA of 512 threads per token row; a thread owns NI quads of four consecutive columns
// (quad tid + 512 i) and keeps their values in registers, with every global load of the row
// issued before the first use (the stage is bound by the latency of its loads, not their bytes).
// The norm gains (constant weights) of the thread's quads are copied into shared memory before the
// wait for the preceding product, so no gain load sits between the reductions.
// The quantisation is norm_quant's: r = (v * (1/rms)) * gain in float32, a = max|r|,
// code = rint(r * (127/a)), factor a/127. Requires the vector lengths to be multiples of 4 and
// at most 4 * 512 * NI = 8192.
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace mmf {
namespace drow {

constexpr int kThreads = 512;
constexpr int kNI = 4;                          // quads per thread
constexpr int kMaxK = 4 * kThreads * kNI;       // 8192

enum Mode : int32_t { kQuantIn = 0, kIFG = 1, kO = 2, kGate = 3, kDown = 4 };

struct Args {
  int32_t mode;
  int32_t d;
  int32_t inner;
  float eps;
  mmf_dtype dt;          // activation dtype (x, x1, v, y)
  const int32_t* acc;    // [b][ldacc] integer products of the preceding group (16-byte rows)
  int64_t ldacc;
  const float* deq_in[3];  // [b] factors a/127 of that group's input codes (kIFG: i, f, g)
  const float* sw[3];      // its weight scales
  const void* x;         // kQuantIn: input rows [b][d]
  const void* res;       // kO: x [b][d]; kDown: x1 [b][d]
  float* state;          // kIFG: [b][d] recurrent state, read and overwritten
  const float* gnorm_w;  // kIFG: g_norm gain (nullable = 1)
  void* out;             // kO: x1; kGate: v; kDown: y -- [b][n] in dt
  int32_t ngain;         // quantisations of the produced vector (0: none)
  const float* gain[3];  // their norm gains (nullable = 1)
  int8_t* q[3];          // [b][ldq] codes (columns past the vector's length written as 0)
  int64_t ldq;
  float* deq[3];         // [b] factors a/127
  float* z_tap;          // kIFG debug tap: [b][3d] float32 zi | zf | g (nullable)
  float* h_tap;          // kIFG debug tap: [b][d] float32 h (nullable)
};

// z = float(acc) * ((a/127) * s), the rounding order of the tensor-core epilogue
__device__ __forceinline__ float dr_scale(int32_t acc, float dq) { return __fmul_rn((float)acc, dq); }
__device__ __forceinline__ float dr_round(float v, mmf_dtype dt) {
  return dt == MMF_F32 ? v : __bfloat162float(__float2bfloat16_rn(v));
}
__device__ __forceinline__ float4 ld4(const void* base, int64_t idx, mmf_dtype dt) {
  if (dt == MMF_F32) return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx);
  const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(base) + idx);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xffff0000u));
}
__device__ __forceinline__ void st4(void* base, int64_t idx, mmf_dtype dt, const float (&v)[4]) {
  if (dt == MMF_F32) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + idx) = make_float4(v[0], v[1], v[2], v[3]);
  } else {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(base) + idx) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
  }
}
// Shared-memory gain slots: slot j < ngain holds gain[j], slot ngain the g_norm gain (kIFG), each
// k floats (only the slots of present gains are filled; absent ones read as ones).
__host__ __device__ inline size_t row_stage_smem(int mode, int d, int inner, int ngain) {
  const int k = mode == kGate ? inner : d;
  return (size_t)(ngain + (mode == kIFG ? 1 : 0)) * (size_t)k * sizeof(float);
}

__global__ void __launch_bounds__(kThreads) row_stage_kernel(const Args a) {
  __shared__ float red[32];
  extern __shared__ __align__(16) float gsm[];     // gain slots (row_stage_smem)
  const int64_t r = blockIdx.x;
  const int tid = threadIdx.x;
  const int k = a.mode == kGate ? a.inner : a.d;  // length of the vector to quantise
  const int nq = k >> 2;                           // quads
  // this thread's quads of every present gain (constant weights: copied before the wait)
  for (int j = 0; j <= a.ngain; ++j) {
    const float* src = j < a.ngain ? a.gain[j] : (a.mode == kIFG ? a.gnorm_w : nullptr);
    if (src == nullptr) continue;
#pragma unroll
    for (int i = 0; i < kNI; ++i) {
      const int qd = tid + i * kThreads;
      if (qd < nq) cp_async16(gsm + (size_t)j * k + 4 * qd, src + 4 * qd);
    }
  }
  cp_async_commit();
  // programmatic dependent launch: wait for the preceding product, then let the next product
  // start streaming its weights while this stage runs
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // a gain quad of this thread: from its own copy in shared memory (ones when absent)
  auto sg4 = [&](int j, const float* present, int c) {
    return present ? *reinterpret_cast<const float4*>(gsm + (size_t)j * k + c) : make_float4(1.0f, 1.0f, 1.0f, 1.0f);
  };
  const int32_t* acc = a.acc ? a.acc + r * a.ldacc : nullptr;
  float v[kNI][4];
  float ss = 0.0f;
  if (a.mode == kIFG) {
    const int d = a.d;
    const float dqi = a.deq_in[0][r] * a.sw[0][0];
    const float dqf = a.deq_in[1][r] * a.sw[1][0];
    const float dqg = a.deq_in[2][r] * a.sw[2][0];
    int4 ai[kNI], af[kNI], ag[kNI];
    float4 hp[kNI];
#pragma unroll
    for (int i = 0; i < kNI; ++i) {
      const int qd = tid + i * kThreads;
      if (qd < nq) {
        ai[i] = *reinterpret_cast<const int4*>(acc + 4 * qd);
        af[i] = *reinterpret_cast<const int4*>(acc + d + 4 * qd);
        ag[i] = *reinterpret_cast<const int4*>(acc + 2 * d + 4 * qd);
        hp[i] = *reinterpret_cast<const float4*>(a.state + r * d + 4 * qd);
      }
    }
    float sh = 0.0f;
    float g[kNI][4];
#pragma unroll
    for (int i = 0; i < kNI; ++i) {
      const int qd = tid + i * kThreads;
      if (qd < nq) {
        const int32_t xi[4] = {ai[i].x, ai[i].y, ai[i].z, ai[i].w};
        const int32_t xf[4] = {af[i].x, af[i].y, af[i].z, af[i].w};
        const int32_t xg[4] = {ag[i].x, ag[i].y, ag[i].z, ag[i].w};
        const float hprev[4] = {hp[i].x, hp[i].y, hp[i].z, hp[i].w};
        float zi[4], zf[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          zi[e] = dr_scale(xi[e], dqi);
          zf[e] = dr_scale(xf[e], dqf);
          g[i][e] = dr_scale(xg[e], dqg);
          float f, omf;
          hgrn_forget(zf[e], f, omf);
          v[i][e] = f * hprev[e] + siluf_(zi[e]) * omf;
          sh = fmaf(v[i][e], v[i][e], sh);
        }
        *reinterpret_cast<float4*>(a.state + r * d + 4 * qd) = make_float4(v[i][0], v[i][1], v[i][2], v[i][3]);
        if (a.h_tap) *reinterpret_cast<float4*>(a.h_tap + r * d + 4 * qd) = make_float4(v[i][0], v[i][1], v[i][2], v[i][3]);
        if (a.z_tap) {
          float* zt = a.z_tap + r * 3 * (int64_t)d + 4 * qd;
          *reinterpret_cast<float4*>(zt) = make_float4(zi[0], zi[1], zi[2], zi[3]);
          *reinterpret_cast<float4*>(zt + d) = make_float4(zf[0], zf[1], zf[2], zf[3]);
          *reinterpret_cast<float4*>(zt + 2 * (int64_t)d) = make_float4(g[i][0], g[i][1], g[i][2], g[i][3]);
        }
      }
    }
    cp_async_wait<0>();  // this thread's gain copies have landed
    const float rh = nq_rinv(block_sum(sh, red), d, a.eps);
    // g_norm: u = (h * (1/rms(h))) * gnorm_w * SiLU(g)
#pragma unroll
    for (int i = 0; i < kNI; ++i) {
      const int qd = tid + i * kThreads;
      if (qd < nq) {
        const float4 w4 = sg4(a.ngain, a.gnorm_w, 4 * qd);
        const float w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[i][e] = __fmul_rn(__fmul_rn(v[i][e], rh), w[e]) * siluf_(g[i][e]);
          ss = fmaf(v[i][e], v[i][e], ss);
        }
      }
    }
  } else {
    const float dq = a.mode == kQuantIn ? 0.0f : a.deq_in[0][r] * a.sw[0][0];
    int4 x0[kNI], x1[kNI];
    float4 rs[kNI];
#pragma unroll
    for (int i = 0; i < kNI; ++i) {
      const int qd = tid + i * kThreads;
      if (qd < nq) {
        if (a.mode == kQuantIn) {
          rs[i] = ld4(a.x, r * a.d + 4 * qd, a.dt);
        } else {
          x0[i] = *reinterpret_cast<const int4*>(acc + 4 * qd);
          if (a.mode == kGate) x1[i] = *reinterpret_cast<const int4*>(acc + k + 4 * qd);
          else rs[i] = ld4(a.res, r * a.d + 4 * qd, a.dt);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kNI; ++i) {
      const int qd = tid + i * kThreads;
      if (qd < nq) {
        if (a.mode == kQuantIn) {
          v[i][0] = rs[i].x; v[i][1] = rs[i].y; v[i][2] = rs[i].z; v[i][3] = rs[i].w;
        } else if (a.mode == kGate) {
          const int32_t gg[4] = {x0[i].x, x0[i].y, x0[i].z, x0[i].w};
          const int32_t uu[4] = {x1[i].x, x1[i].y, x1[i].z, x1[i].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) v[i][e] = dr_round(siluf_(dr_scale(gg[e], dq)) * dr_scale(uu[e], dq), a.dt);
          st4(a.out, r * k + 4 * qd, a.dt, v[i]);
        } else {
          const int32_t aa[4] = {x0[i].x, x0[i].y, x0[i].z, x0[i].w};
          const float rr[4] = {rs[i].x, rs[i].y, rs[i].z, rs[i].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) v[i][e] = dr_round(dr_scale(aa[e], dq) + rr[e], a.dt);
          st4(a.out, r * k + 4 * qd, a.dt, v[i]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) ss = fmaf(v[i][e], v[i][e], ss);
      }
    }
  }
  if (a.ngain == 0) return;
  cp_async_wait<0>();  // this thread's gain copies have landed
  const float rf = nq_rinv(block_sum(ss, red), k, a.eps);
  for (int j = 0; j < a.ngain; ++j) {
    const float* gn = a.gain[j];
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < kNI; ++i) {
      const int qd = tid + i * kThreads;
      if (qd < nq) {
        const float4 w4 = sg4(j, gn, 4 * qd);
        const float w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) am = fmaxf(am, fabsf(__fmul_rn(__fmul_rn(v[i][e], rf), w[e])));
      }
    }
    am = fmaxf(block_max(am, red), 1e-5f);
    const float sx = q127_over(am);
    int8_t* qrow = a.q[j] + r * a.ldq;
#pragma unroll
    for (int i = 0; i < kNI; ++i) {
      const int qd = tid + i * kThreads;
      if (qd < nq) {
        const float4 w4 = sg4(j, gn, 4 * qd);
        const float w[4] = {w4.x, w4.y, w4.z, w4.w};
        uint32_t qb[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) qb[e] = q8_bits(__fmul_rn(__fmul_rn(__fmul_rn(v[i][e], rf), w[e]), sx));
        *reinterpret_cast<uint32_t*>(qrow + 4 * qd) = pack4_lo_bytes(qb[0], qb[1], qb[2], qb[3]);
      }
    }
    for (int c = k + 4 * tid; c < a.ldq; c += 4 * kThreads) *reinterpret_cast<uint32_t*>(qrow + c) = 0u;
    if (tid == 0) a.deq[j][r] = over_127(am);
  }
}

}  // namespace drow
}  // namespace mmf
