// decode.cuh -- K8: fused decode projections for up to 8 token rows (one autoregressive step).
//
// One decode step of a block is four launches of dec_proj_kernel, one per projection group, each
// with its producer and consumer steps fused in:
//   kIFG   RMSNorm + int8 quantisation of x with the i/f/g gains (prologue), the i, f and g
//          products, and the HGRN gates + one recurrence step h = f h_prev + i on the carried
//          state (epilogue; writes h and g in float32);
//   kO     g_norm u = RMSNorm(h) * w_g * SiLU(g) and o_proj's RMSNorm + quantisation (prologue),
//          o_proj and the residual x1 = x + o (epilogue);
//   kGate  gate_proj's RMSNorm + quantisation of x1, gate and up rows of the same channels, and
//          v = SiLU(gate) * up (epilogue);
//   kDown  down_proj's RMSNorm + quantisation of v, down_proj and y = x1 + down (epilogue).
// Each CTA owns a contiguous range of output channels. Its first thread starts bulk copies of
// the input rows and their norm gains, then of the CTA's packed weight rows, into shared memory
// (two barriers);
// while the weights stream in, the CTA quantises the input rows itself -- every CTA computes the
// same codes, in the arithmetic of norm_quant_vec_kernel -- and each half-warp then forms whole
// output channels (one at a time, four from four token rows on): its 16 lanes stride over 32-code
// (8-byte) pieces of the weight rows (expanded with byte permutes), dp4a them against the codes,
// and reduce per (matrix, channel, row) with shuffles inside the half-warp.
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace mmf {
namespace dec {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxRows = 8;            // token rows per launch
constexpr int kStageRows = 2;          // input rows staged in shared memory up to this count
// per-row reduction scratch: two rounds of sum-of-squares partials [round][warp][row], maxima
// partials [warp][gain][row]
constexpr int kRedFloats = (2 * kWarps + 3 * kWarps) * kMaxRows;
constexpr int kMaxSmem = 200 * 1024;   // dynamic shared memory budget per CTA

enum Mode : int32_t { kIFG = 0, kO = 1, kGate = 2, kDown = 3 };

struct Args {
  int32_t mode;
  int32_t b;              // token rows (1..8)
  int32_t k;              // input features
  int32_t kw;             // packed words per weight row (4 * ceil(k / 64))
  int32_t nout;           // output channels
  int32_t chan_per_cta;
  int32_t nmat;           // weight rows per channel: kIFG 3 (i, f, g), kGate 2 (gate, up), else 1
  int32_t ngain;          // quantisations of the input: kIFG 3 (one per gain), else 1
  float eps;
  const uint32_t* w[3];   // weight row c of matrix j: w[j] + (row_off[j] + c) * kw
  int32_t row_off[3];
  const float* sw[3];     // weight scales
  const float* gain[3];   // RMSNorm gains of the input (kIFG: i, f, g; else the projection's)
  const void* x;          // input rows [b][k]: x (kIFG), x1 (kGate), v (kDown), dtype xdt
  mmf_dtype xdt;
  const float* h;         // kO: h [b][k] float32
  const float* gin;       // kO: g [b][k] float32
  const float* gnorm_w;   // kO: g_norm gain (nullable = 1)
  const void* res;        // kO / kDown: residual [b][nout], dtype ydt
  void* y;                // kIFG: h float32; kO: x1; kGate: v; kDown: y -- [b][nout]
  mmf_dtype ydt;
  float* g_out;           // kIFG: g [b][nout] float32
  float* state;           // kIFG: recurrent state [b][nout] float32, read and overwritten
  uint32_t wait_limit_us;
  // debug taps (null on the timed path): CTA 0 copies the codes it formed, [gain][row][k] int8,
  // and the factors a/127, [gain][row]; kIFG also writes zi, zf and g as [row][3 * nout] float32
  int8_t* q_tap;
  float* deq_tap;
  float* z_tap;
};

// Shared-memory layout of one CTA: weight rows, norm gains (ngain vectors of k floats; kO also
// the g_norm gain), the g_norm output u (kO only, [b][k] float32), the codes, factors, scratch.
struct Smem {
  size_t w_bytes, gain_off, u_off, x_off, q_off, q_bytes, deq_off, red_off, tot_off, bar_off, total;
};
__host__ __device__ inline Smem smem_layout(int mode, int nmat, int chan_per_cta, int kw, int k, int ngain, int b) {
  Smem s;
  s.w_bytes = (size_t)nmat * chan_per_cta * kw * 4;
  s.gain_off = (s.w_bytes + 127) & ~(size_t)127;
  const int ngv = ngain + (mode == kO ? 1 : 0);
  s.u_off = (s.gain_off + (size_t)ngv * k * 4 + 127) & ~(size_t)127;
  const size_t u_bytes = mode == kO ? (size_t)b * k * 4 : 0;
  // the input rows, copied in with the gains when there are at most kStageRows of them: x, x1
  // or v (<= 4 bytes per value); kO: h and g. More rows are read from global memory.
  s.x_off = (s.u_off + u_bytes + 127) & ~(size_t)127;
  const size_t x_bytes = b <= kStageRows ? (size_t)(mode == kO ? 2 : 1) * b * k * 4 : 0;
  s.q_off = (s.x_off + x_bytes + 127) & ~(size_t)127;
  s.q_bytes = (size_t)ngain * b * kw * 16;   // codes of the padded K, [gain][row][piece][chunk]
  s.deq_off = (s.q_off + s.q_bytes + 15) & ~(size_t)15;
  s.red_off = s.deq_off + 3 * kMaxRows * sizeof(float);
  s.tot_off = s.red_off + kRedFloats * sizeof(float);  // [matrix][channel][row] int32
  s.bar_off = (s.tot_off + (size_t)nmat * chan_per_cta * b * 4 + 7) & ~(size_t)7;
  s.total = s.bar_off + 16;   // two mbarriers: gains, weights
  return s;
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Input value k of token row r as the projection's RMSNorm sees it: the staged row itself, or for
// kO the g_norm output u; both in shared memory.
template <mmf_dtype XT>
__device__ __forceinline__ void in8(const Args& a, const float* us, const void* xs, int r, int kk, float (&o)[8]) {
  if (a.mode == kO) {
    const float4 p = *reinterpret_cast<const float4*>(us + (size_t)r * a.k + kk);
    const float4 q = *reinterpret_cast<const float4*>(us + (size_t)r * a.k + kk + 4);
    o[0] = p.x; o[1] = p.y; o[2] = p.z; o[3] = p.w;
    o[4] = q.x; o[5] = q.y; o[6] = q.z; o[7] = q.w;
  } else {
    load8<XT>(xs, (int64_t)r * a.k + kk, o);
  }
}
__device__ __forceinline__ void sm8(const float* p, float (&o)[8]) {
  const float4 x = *reinterpret_cast<const float4*>(p);
  const float4 y = *reinterpret_cast<const float4*>(p + 4);
  o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
  o[4] = y.x; o[5] = y.y; o[6] = y.z; o[7] = y.w;
}

// The residual, read through L2 (it was written by an earlier launch on other SMs).
__device__ __forceinline__ float res_as_float(const void* base, int64_t idx, mmf_dtype dt) {
  if (dt == MMF_F32) return __ldcg(reinterpret_cast<const float*>(base) + idx);
  const unsigned short u = __ldcg(reinterpret_cast<const unsigned short*>(base) + idx);
  return __uint_as_float((uint32_t)u << 16);
}

// Shared-memory pieces of one CTA for one projection group: the weight rows (requested before the
// phase, possibly during the previous one), the gains, u, the staged input rows, the codes, the
// factors and scratch, and the two barriers with the parity each completes next.
struct Bufs {
  uint32_t* wsm;
  float* gains;
  float* us;
  uint8_t* xsm;
  int8_t* qs;
  float* deqs;
  float* red;
  int32_t* tots;      // [matrix][channel][row] integer products of the CTA's channels
  uint64_t* bar_in;   // input rows + gains
  uint64_t* bar_w;    // weight rows
  uint32_t par_in, par_w;
};

// Thread 0: request this CTA's weight rows of the group (channels cta * chan_per_cta ...).
__device__ __forceinline__ void dec_issue_weights(const Args& a, uint32_t* wsm, uint64_t* bar_w, int cta) {
  const int c0 = cta * a.chan_per_cta;
  int nc = a.nout - c0 < a.chan_per_cta ? a.nout - c0 : a.chan_per_cta;
  if (nc < 0) nc = 0;  // (defensive: the grid never has a CTA past the last channel)
  const uint32_t row_bytes = (uint32_t)a.kw * 4u;
  mbar_arrive_expect_tx(bar_w, (uint32_t)a.nmat * (uint32_t)nc * row_bytes);
  if (nc > 0)
    for (int j = 0; j < a.nmat; ++j)
      bulk_load(wsm + (size_t)j * a.chan_per_cta * a.kw, a.w[j] + ((int64_t)a.row_off[j] + c0) * a.kw,
                (uint32_t)nc * row_bytes, bar_w);
}

// One projection group on one CTA: input rows and gains into shared memory, then the weight rows
// (all requested by thread 0 at the start), the codes of every input row, the products and the
// fused epilogue.
// Returns false when a bounded wait gave up (the copies in flight are drained first).
template <mmf_dtype XT, int NB>
__device__ __forceinline__ bool dec_phase(const Args& a, const Bufs& B, int cta) {
  float* gains = B.gains;
  float* us = B.us;
  // input rows: staged in shared memory (kO: h, then g) or read in place
  constexpr bool kStage = NB <= kStageRows;
  uint8_t* xsm = B.xsm;
  const void* xs = kStage ? static_cast<const void*>(xsm) : a.x;
  const float* hs = kStage ? reinterpret_cast<const float*>(xsm) : a.h;
  const float* gs = kStage ? hs + (size_t)a.b * a.k : a.gin;
  int8_t* qs = B.qs;
  float* deqs = B.deqs;
  float* red = B.red;
  uint32_t* wsm = B.wsm;
  const int c0 = cta * a.chan_per_cta;
  const int nc = a.nout - c0 < a.chan_per_cta ? a.nout - c0 : a.chan_per_cta;
  const uint32_t gbytes = (uint32_t)a.k * 4u;
  const bool has_gw = a.mode == kO && a.gnorm_w != nullptr;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ng = a.ngain;

  // 1. the input rows and their norm gains into shared memory (absent gains are ones)
  if (threadIdx.x == 0) {
    const uint32_t xbytes = kStage ? (uint32_t)a.b * (uint32_t)a.k * (a.mode == kO ? 4u : (XT == MMF_F32 ? 4u : 2u)) : 0u;
    uint32_t tx = (a.mode == kO ? 2u : 1u) * xbytes;
    for (int j = 0; j < ng; ++j) tx += a.gain[j] ? gbytes : 0u;
    if (has_gw) tx += gbytes;
    mbar_arrive_expect_tx(B.bar_in, tx);
    if (kStage && a.mode == kO) {
      bulk_load(xsm, a.h, xbytes, B.bar_in);
      bulk_load(xsm + xbytes, a.gin, xbytes, B.bar_in);
    } else if (kStage) {
      bulk_load(xsm, a.x, xbytes, B.bar_in);
    }
    for (int j = 0; j < ng; ++j)
      if (a.gain[j]) bulk_load(gains + (size_t)j * a.k, a.gain[j], gbytes, B.bar_in);
    if (has_gw) bulk_load(gains + (size_t)ng * a.k, a.gnorm_w, gbytes, B.bar_in);
    // the weight rows after the inputs: the prologue waits only for the inputs, and copies
    // requested first arrive first (requesting the weights first cost 5-7% of a decode step)
    dec_issue_weights(a, B.wsm, B.bar_w, cta);
  }
  for (int j = 0; j < ng + (a.mode == kO ? 1 : 0); ++j) {
    const bool absent = j < ng ? a.gain[j] == nullptr : !has_gw;
    if (absent)
      for (int t = threadIdx.x; t < a.k; t += kThreads) gains[(size_t)j * a.k + t] = 1.0f;
  }
  // (the decision is CTA-uniform, so every thread takes the same barriers afterwards; a
  //  timed-out wait drains both copies before the CTA leaves: shared memory must outlive them)
  volatile int abort_flag = 0;
  auto wait_or_leave = [&](uint64_t* bar, uint32_t par) {
    const bool mine = mbar_wait_bounded(bar, par, a.wait_limit_us, &abort_flag);
    if (!__syncthreads_or(mine ? 0 : 1)) return true;
    const int64_t t0 = clock64();
    while (!mbar_try_wait(B.bar_in, B.par_in) && clock64() - t0 < 1000000ll * kCyclesPerUs) {
    }
    const int64_t t1 = clock64();
    while (!mbar_try_wait(B.bar_w, B.par_w) && clock64() - t1 < 1000000ll * kCyclesPerUs) {
    }
    return false;
  };
  if (!wait_or_leave(B.bar_in, B.par_in)) return false;

  // 2. prologue: the codes of every input row (the same in every CTA). The row loops run over
  //    the compile-time count NB inside the chunk loops, so the loads of all rows are in flight
  //    together (the rows are read in place when there are more than kStageRows of them).
  const int nck = a.k >> 3;
  const int kq = a.kw * 16;
  // every round leaves one partial per warp and row; after one barrier each thread combines
  // them itself (same order everywhere), so no second barrier is needed
  float* ssp = red;                                   // [round][warp][row]
  float* amp = red + 2 * kWarps * kMaxRows;           // [warp][gain][row]
  float rf[NB], rfh[NB];
  // 2a. mean squares of every row (kO: of h, then u = h / rms(h) * w_g * SiLU(g) into shared
  //     memory and its mean squares)
  for (int pass = 0; pass < (a.mode == kO ? 2 : 1); ++pass) {
    float ss[NB];
#pragma unroll
    for (int r = 0; r < NB; ++r) ss[r] = 0.0f;
    for (int c = threadIdx.x; c < nck; c += kThreads) {
      if (a.mode == kO && pass == 1) {
        float w8[8];
        sm8(gains + (size_t)ng * a.k + 8 * c, w8);
#pragma unroll
        for (int r = 0; r < NB; ++r) {
          float v[8], g[8];
          load8<MMF_F32>(hs, (int64_t)r * a.k + 8 * c, v);
          load8<MMF_F32>(gs, (int64_t)r * a.k + 8 * c, g);
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = __fmul_rn(__fmul_rn(v[e], rfh[r]), w8[e]) * siluf_(g[e]);
          float* up = us + (size_t)r * a.k + 8 * c;
          *reinterpret_cast<float4*>(up) = make_float4(v[0], v[1], v[2], v[3]);
          *reinterpret_cast<float4*>(up + 4) = make_float4(v[4], v[5], v[6], v[7]);
#pragma unroll
          for (int e = 0; e < 8; ++e) ss[r] = fmaf(v[e], v[e], ss[r]);
        }
      } else {
        float v[NB][8];
#pragma unroll
        for (int r = 0; r < NB; ++r) {
          if (a.mode == kO) load8<MMF_F32>(hs, (int64_t)r * a.k + 8 * c, v[r]);
          else load8<XT>(xs, (int64_t)r * a.k + 8 * c, v[r]);
        }
#pragma unroll
        for (int r = 0; r < NB; ++r)
#pragma unroll
          for (int e = 0; e < 8; ++e) ss[r] = fmaf(v[r][e], v[r][e], ss[r]);
      }
    }
    float* part = ssp + pass * kWarps * kMaxRows;
#pragma unroll
    for (int r = 0; r < NB; ++r) {
      const float t = warp_sum(ss[r]);
      if (lane == 0) part[warp * kMaxRows + r] = t;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < NB; ++r) {
      float t = 0.0f;
      for (int w = 0; w < kWarps; ++w) t += part[w * kMaxRows + r];
      if (a.mode == kO && pass == 0) rfh[r] = nq_rinv(t, a.k, a.eps);
      else rf[r] = nq_rinv(t, a.k, a.eps);
    }
  }
  // 2b. maxima of |r| = |v / rms * gain| per (gain, row)
  for (int j = 0; j < ng; ++j) {
    float am[NB];
#pragma unroll
    for (int r = 0; r < NB; ++r) am[r] = 0.0f;
    for (int c = threadIdx.x; c < nck; c += kThreads) {
      float gg[8];
      sm8(gains + (size_t)j * a.k + 8 * c, gg);
      float v[NB][8];
#pragma unroll
      for (int r = 0; r < NB; ++r) in8<XT>(a, us, xs, r, 8 * c, v[r]);
#pragma unroll
      for (int r = 0; r < NB; ++r) {
#pragma unroll
        for (int e = 0; e < 8; ++e) am[r] = fmaxf(am[r], fabsf(__fmul_rn(__fmul_rn(v[r][e], rf[r]), gg[e])));
      }
    }
#pragma unroll
    for (int r = 0; r < NB; ++r) {
      const float t = warp_max(am[r]);
      if (lane == 0) amp[(warp * 3 + j) * kMaxRows + r] = t;
    }
  }
  __syncthreads();
  // 127/a per (gain, row), formed by every thread; the factors a/127 for the epilogue
  float sx[3][NB];
  for (int j = 0; j < ng; ++j) {
#pragma unroll
    for (int r = 0; r < NB; ++r) {
      float t = 0.0f;
      for (int w = 0; w < kWarps; ++w) t = fmaxf(t, amp[(w * 3 + j) * kMaxRows + r]);
      t = fmaxf(t, 1e-5f);
      const float q = q127_over(t);
      if (j == 0) sx[0][r] = q;
      else if (j == 1) sx[1][r] = q;
      else sx[2][r] = q;
      if (threadIdx.x == 0) deqs[j * kMaxRows + r] = over_127(t);
    }
  }
  // 2c. codes, piece-major: code k of (gain j, row r) at
  //     qs + (j * b + r) * kq + ((k % 64) / 16) * (kq / 4) + (k / 64) * 16 + k % 16
  for (int j = 0; j < ng; ++j) {
    for (int c = threadIdx.x; c < nck; c += kThreads) {
      float gg[8];
      sm8(gains + (size_t)j * a.k + 8 * c, gg);
      float v[NB][8];
#pragma unroll
      for (int r = 0; r < NB; ++r) in8<XT>(a, us, xs, r, 8 * c, v[r]);
      const int kk = 8 * c;
#pragma unroll
      for (int r = 0; r < NB; ++r) {
        const float sxr = j == 0 ? sx[0][r] : (j == 1 ? sx[1][r] : sx[2][r]);
        uint32_t q[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) q[e] = q8_bits(__fmul_rn(__fmul_rn(__fmul_rn(v[r][e], rf[r]), gg[e]), sxr));
        int8_t* qrow = qs + (size_t)(j * NB + r) * kq;
        *reinterpret_cast<uint2*>(qrow + ((kk & 63) >> 4) * (kq >> 2) + (kk >> 6) * 16 + (kk & 15)) =
            make_uint2(pack4_lo_bytes(q[0], q[1], q[2], q[3]), pack4_lo_bytes(q[4], q[5], q[6], q[7]));
      }
    }
  }
  __syncthreads();
  if (a.q_tap != nullptr && cta == 0) {
    // the codes every CTA formed, unscrambled from the piece-major layout
    for (int j = 0; j < ng; ++j)
      for (int e = threadIdx.x; e < NB * a.k; e += kThreads) {
        const int r = e / a.k, kk = e - r * a.k;
        a.q_tap[((size_t)j * NB + r) * a.k + kk] =
            qs[(size_t)(j * NB + r) * kq + ((kk & 63) >> 4) * (kq >> 2) + (kk >> 6) * 16 + (kk & 15)];
      }
    if (threadIdx.x < ng * NB) a.deq_tap[threadIdx.x] = deqs[(threadIdx.x / NB) * kMaxRows + threadIdx.x % NB];
  }

  if (!wait_or_leave(B.bar_w, B.par_w)) return false;

  // 3. products: work items are (group of kCpw channels, matrix) pairs, spread evenly over the
  //    half-warps; a half-warp's 16 lanes stride over 32-code (8-byte) pieces of the channels'
  //    weight rows, load the codes of the NB token rows for a piece once and dp4a them against
  //    all kCpw rows in two independent chains (NB = b is a compile-time count, so no work is
  //    issued for absent rows). Lane r of the half leaves the total of token row r in shared
  //    memory. Both halves of a warp run the same trip counts, so the shuffles stay uniform.
  constexpr int kCpw = NB >= 4 ? 4 : 1;
  const int npc = a.kw >> 1;              // 8-byte pieces per weight row
  const int hw = lane >> 4, hl = lane & 15;
  const int ngroups = (nc + kCpw - 1) / kCpw;
  const int nitems = ngroups * a.nmat;
  int32_t* tots = B.tots;                 // [matrix][channel][row]
  for (int ib = warp * 2; ib < nitems; ib += kWarps * 2) {
    const int it = ib + hw;
    const bool live = it < nitems;
    const int m = live ? it / ngroups : 0;
    const int cg = live ? (it - m * ngroups) * kCpw : nc;  // first channel of the group
    const int gsel = ng == 3 ? m : 0;
    int acc0[kCpw][NB], acc1[kCpw][NB];
    auto& acc1r = NB <= 2 ? acc1 : acc0;  // two chains only where the registers allow it
#pragma unroll
    for (int c = 0; c < kCpw; ++c)
#pragma unroll
      for (int r = 0; r < NB; ++r) acc0[c][r] = acc1[c][r] = 0;
    const uint2* wrow = reinterpret_cast<const uint2*>(wsm + ((size_t)m * a.chan_per_cta + cg) * a.kw);
    const int8_t* qg = qs + (size_t)gsel * NB * kq;
#pragma unroll 2
    for (int pc = hl; pc < npc; pc += 16) {
      const int8_t* qc = qg + (pc >> 1) * 16 + (pc & 1) * 2 * (kq >> 2);  // 64-code chunk, piece pair
      uint4 av[NB][2];
#pragma unroll
      for (int r = 0; r < NB; ++r)
#pragma unroll
        for (int pp = 0; pp < 2; ++pp) av[r][pp] = *reinterpret_cast<const uint4*>(qc + (size_t)r * kq + pp * (kq >> 2));
#pragma unroll
      for (int c = 0; c < kCpw; ++c) {
        if (cg + c < nc) {
          const uint2 wv = wrow[(size_t)c * (a.kw >> 1) + pc];
          uint32_t e[8];
          expand_word(wv.x, e + 0);
          expand_word(wv.y, e + 4);
#pragma unroll
          for (int r = 0; r < NB; ++r) {
            acc0[c][r] = __dp4a((int)e[0], (int)av[r][0].x, acc0[c][r]);
            acc1r[c][r] = __dp4a((int)e[4], (int)av[r][1].x, acc1r[c][r]);
            acc0[c][r] = __dp4a((int)e[1], (int)av[r][0].y, acc0[c][r]);
            acc1r[c][r] = __dp4a((int)e[5], (int)av[r][1].y, acc1r[c][r]);
            acc0[c][r] = __dp4a((int)e[2], (int)av[r][0].z, acc0[c][r]);
            acc1r[c][r] = __dp4a((int)e[6], (int)av[r][1].z, acc1r[c][r]);
            acc0[c][r] = __dp4a((int)e[3], (int)av[r][0].w, acc0[c][r]);
            acc1r[c][r] = __dp4a((int)e[7], (int)av[r][1].w, acc1r[c][r]);
          }
        }
      }
    }
#pragma unroll
    for (int c = 0; c < kCpw; ++c) {
#pragma unroll
      for (int r = 0; r < NB; ++r) {
        int sum = NB <= 2 ? acc0[c][r] + acc1[c][r] : acc0[c][r];
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (hl == r && cg + c < nc) tots[((size_t)m * a.chan_per_cta + cg + c) * NB + r] = sum;
      }
    }
  }
  __syncthreads();

  // 4. epilogue: one thread per (channel, token row) of the CTA
  for (int idx = threadIdx.x; idx < nc * NB; idx += kThreads) {
    const int cl = idx / NB, r = idx - cl * NB;
    const int64_t o = (int64_t)r * a.nout + c0 + cl;
    auto zof = [&](int m) {
      const int gsel = ng == 3 ? m : 0;
      const int tot = tots[((size_t)m * a.chan_per_cta + cl) * NB + r];
      return __fmul_rn((float)tot, __fmul_rn(deqs[gsel * kMaxRows + r], a.sw[m][0]));
    };
    if (a.mode == kIFG) {
      // f = sigmoid(zf), i = SiLU(zi) * (1 - f), h = f * h_prev + i
      const float zi = zof(0), zf = zof(1), zg = zof(2);
      float f, omf;
      hgrn_forget(zf, f, omf);
      const float iv = siluf_(zi) * omf;
      const float hv = f * a.state[o] + iv;
      a.state[o] = hv;
      reinterpret_cast<float*>(a.y)[o] = hv;
      a.g_out[o] = zg;
      if (a.z_tap != nullptr) {
        float* zt = a.z_tap + (int64_t)r * 3 * a.nout + c0 + cl;
        zt[0] = zi;
        zt[a.nout] = zf;
        zt[2 * (int64_t)a.nout] = zg;
      }
    } else if (a.mode == kGate) {
      store_from_float(a.y, o, a.ydt, siluf_(zof(0)) * zof(1));
    } else {
      store_from_float(a.y, o, a.ydt, zof(0) + res_as_float(a.res, o, a.ydt));
    }
  }
  return true;
}

// One projection group per launch. The kernel runs once per SM for a few microseconds, so its
// instructions are fetched cold: the code is kept compact (runtime loops over gains and
// matrices; per-row statistics in shared memory) rather than unrolled.
template <mmf_dtype XT, int NB>
__global__ void __launch_bounds__(kThreads) dec_proj_kernel(const __grid_constant__ Args a) {
  extern __shared__ __align__(128) uint8_t sm[];
  const Smem L = smem_layout(a.mode, a.nmat, a.chan_per_cta, a.kw, a.k, a.ngain, a.b);
  Bufs B;
  B.wsm = reinterpret_cast<uint32_t*>(sm);
  B.gains = reinterpret_cast<float*>(sm + L.gain_off);
  B.us = reinterpret_cast<float*>(sm + L.u_off);
  B.xsm = sm + L.x_off;
  B.qs = reinterpret_cast<int8_t*>(sm + L.q_off);
  B.deqs = reinterpret_cast<float*>(sm + L.deq_off);
  B.red = reinterpret_cast<float*>(sm + L.red_off);
  B.tots = reinterpret_cast<int32_t*>(sm + L.tot_off);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L.bar_off);
  B.bar_in = &bar[0];
  B.bar_w = &bar[1];
  B.par_in = 0u;
  B.par_w = 0u;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_fence_init();
  }
  __syncthreads();
  dec_phase<XT, NB>(a, B, blockIdx.x);
}

}  // namespace dec
}  // namespace mmf
