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
};

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
      v = siluf_(gate) * up;
    } else {
      const double hv = load_as_float(a.x, row * a.ldx + c, a.xdt);
      const float gv = load_as_float(a.g, row * a.ldg + c, a.gdt);
      v = (float)(hv * rinv_h * (double)(a.gw ? a.gw[c] : 1.0f)) * siluf_(gv);
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
    const float sx = __fdiv_rn(127.0f, amax);
    int8_t* qrow = a.q[j] + row * a.ldq;
    for (int c = threadIdx.x; c < a.ldq; c += blockDim.x) {
      int8_t code = 0;
      if (c < k) {
        const float r = (float)((double)vrow[c] * rinv * (double)(gn ? gn[c] : 1.0f));
        code = (int8_t)fminf(fmaxf(rintf(__fmul_rn(r, sx)), -127.0f), 127.0f);
      }
      qrow[c] = code;
    }
    if (threadIdx.x == 0) a.deq[j][row] = __fdiv_rn(amax, 127.0f);
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

// y = acc * deq[row] * s (+ residual), plus the optional raw accumulator.
__device__ __forceinline__ void bitlinear_epilogue(const GemmSeg& s, mmf_dtype ydt, int64_t row,
                                                   int32_t col, int32_t acc, float sw) {
  if (s.acc) s.acc[row * s.ldacc + col] = acc;
  float z = (float)acc * (s.deq[row] * sw);  // same rounding order as the tensor-core epilogue
  if (s.res) z += load_as_float(s.res, row * s.ldres + s.rescol + col, ydt);
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
  // stage activations
  for (int idx = threadIdx.x; idx < mt * nchunk * 4; idx += blockDim.x) {
    const int j = idx / (nchunk * 4);
    const int rem = idx - j * nchunk * 4;
    const int c = rem >> 2, p = rem & 3;
    sact[j * nchunk * 4 + p * nchunk + c] =
        *reinterpret_cast<const uint4*>(s.q + (m0 + j) * a.ldq + c * 64 + p * 16);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 3, l8 = lane & 7;
  const float sw = s.sw[0];
  for (int base = blockIdx.x * 32 + warp * 4; base < s.n; base += gridDim.x * 32) {
    const int n = base + grp;
    const bool valid = n < s.n;
    int acc[kSimtMT];
#pragma unroll
    for (int j = 0; j < kSimtMT; ++j) acc[j] = 0;
    const uint4* wrow = reinterpret_cast<const uint4*>(s.codes + (int64_t)(valid ? n : 0) * a.kw);
    for (int c = l8; c < nchunk; c += 8) {
      uint4 wv = make_uint4(0u, 0u, 0u, 0u);
      if (valid) wv = __ldg(wrow + c);
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
// K4: HGRN scan with fused gates
// =============================================================================================
// CTA = 32 channels (lanes) x kScanWarps warps. The sequence is processed in segments of
// kScanWarps * kScanL steps; warp w owns steps [w*L, (w+1)*L) of a segment. Each warp folds its
// steps into an affine map (A, B) (h -> A h + B), the maps are published in shared memory, each
// warp composes the maps of the warps before it onto the segment's carry, then replays its own
// steps sequentially from that carry and stores h.
constexpr int kScanWarps = 16;
constexpr int kScanL = 8;

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
};

__global__ void __launch_bounds__(kScanWarps * 32) hgrn_scan_kernel(const ScanArgs a) {
  __shared__ float sA[kScanWarps][32];
  __shared__ float sB[kScanWarps][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t ch = (int64_t)blockIdx.x * 32 + lane;
  const bool valid = ch < (int64_t)a.b * a.d;
  const int64_t bi = valid ? ch / a.d : 0;
  const int64_t c = valid ? ch - bi * a.d : 0;
  const int64_t zbase = bi * a.t * a.zstride + c;
  const int64_t hbase = bi * a.t * a.d + c;
  float carry = (valid && a.h0) ? a.h0[bi * a.d + c] : 0.0f;
  for (int64_t seg0 = 0; seg0 < a.t; seg0 += kScanWarps * kScanL) {
    const int64_t t0 = seg0 + (int64_t)warp * kScanL;
    float f[kScanL], in[kScanL];
#pragma unroll
    for (int s = 0; s < kScanL; ++s) {
      const int64_t t = t0 + s;
      if (valid && t < a.t) {
        const float zf = load_as_float(a.zf, zbase + t * a.zstride, a.zdt);
        const float zi = load_as_float(a.zi, zbase + t * a.zstride, a.zdt);
        const float fg = sigmoidf_(zf);
        f[s] = fg;
        in[s] = siluf_(zi) * (1.0f - fg);
      } else {
        f[s] = 1.0f;  // identity step
        in[s] = 0.0f;
      }
    }
    float A = 1.0f, B = 0.0f;
#pragma unroll
    for (int s = 0; s < kScanL; ++s) {
      A = f[s] * A;
      B = f[s] * B + in[s];
    }
    sA[warp][lane] = A;
    sB[warp][lane] = B;
    __syncthreads();
    float h = carry;
    for (int w = 0; w < warp; ++w) h = sA[w][lane] * h + sB[w][lane];
#pragma unroll
    for (int s = 0; s < kScanL; ++s) {
      h = f[s] * h + in[s];
      const int64_t t = t0 + s;
      if (valid && t < a.t) store_from_float(a.h, hbase + t * a.d, a.hdt, h);
    }
    float cnext = carry;
    for (int w = 0; w < kScanWarps; ++w) cnext = sA[w][lane] * cnext + sB[w][lane];
    carry = cnext;
    __syncthreads();
  }
  if (valid && warp == 0 && a.h_last) a.h_last[bi * a.d + c] = carry;
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

}  // namespace mmf
