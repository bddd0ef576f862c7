// validate.cuh -- integrity check of a packed ternary matrix.
//
// In the packed format a 2-bit field is 00 (0), 01 (+1) or 11 (-1); 10 is unused, and the fields
// of the padding columns k .. 16 * row_words - 1 of each row are 00. A word holds 16 fields: the
// code of column 16 w + j (j = 4 quad + lane) sits at bit 16 (quad >> 1) + 2 (quad & 1) + 4 lane.
// The kernel counts, over every word, the real-column fields holding 10 and the nonzero padding
// fields (each malformed field once), and adds the total to a device counter: any nonzero count means the codes were corrupted (or never
// packed by mmf_pack_ternary).
#pragma once

#include "common.cuh"

namespace mmf {
namespace validate {

constexpr int kThreads = 256;

// Mask of the low bits of the fields of columns j >= jmin in one word (jmin in [0, 16]).
__device__ __forceinline__ uint32_t fields_from(int jmin) {
  uint32_t m = 0u;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int quad = j >> 2, lane = j & 3;
    if (j >= jmin) m |= 1u << (16 * (quad >> 1) + 2 * (quad & 1) + 4 * lane);
  }
  return m;
}

__global__ void __launch_bounds__(kThreads) validate_packed_kernel(const uint32_t* __restrict__ codes, int32_t n,
                                                                   int32_t k, int32_t kw,
                                                                   unsigned long long* __restrict__ bad) {
  const int64_t total = (int64_t)n * kw;
  unsigned long long count = 0ull;
  for (int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x; e < total; e += (int64_t)gridDim.x * kThreads) {
    const uint32_t w = codes[e];
    const int col0 = (int)(e % kw) * 16;
    const uint32_t lo = w & 0x55555555u, hi = (w >> 1) & 0x55555555u;
    // fields of padding columns (every one must be 00; each nonzero one counts once, a 10 there
    // included) and of real columns (a 10 counts)
    const uint32_t pad = col0 + 16 > k ? fields_from(k - col0 < 0 ? 0 : k - col0) : 0u;
    count += __popc(hi & ~lo & ~pad) + __popc((lo | hi) & pad);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) count += __shfl_xor_sync(0xffffffffu, count, o);
  if ((threadIdx.x & 31) == 0 && count) atomicAdd(bad, count);
}

}  // namespace validate
}  // namespace mmf
