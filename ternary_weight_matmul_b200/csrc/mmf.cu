// mmf.cu -- C ABI of libmmf (declared in include/mmf.h): argument validation, workspace layout,
// engine dispatch and launches. All kernels live in the headers included below (one translation
// unit, so the device error flag is shared without relocatable device code).
#include <cudaTypedefs.h>

#include <algorithm>
#include <utility>
#include <cstdarg>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "decode.cuh"
#include "decode_rows.cuh"
#include "gemm_bf16.cuh"
#include "gemm_skinny.cuh"
#include "gemm_tc.cuh"
#include "head.cuh"
#include "hgrn2.cuh"
#include "backward.cuh"
#include "validate.cuh"
#include "kernels.cuh"

using namespace mmf;

namespace {

thread_local std::string g_last_error;
std::atomic<int> g_gemm_path{MMF_GEMM_AUTO};
std::atomic<int> g_decode_path{MMF_DECODE_AUTO};
constexpr uint32_t kDefaultWaitLimit = 2000000u;  // microseconds
std::atomic<uint32_t> g_wait_limit{kDefaultWaitLimit};

mmf_status fail(mmf_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
mmf_status fail(mmf_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

#define MMF_CHECK_ARG(cond, ...)                                   \
  do {                                                             \
    if (!(cond)) return fail(MMF_ERR_INVALID_ARG, __VA_ARGS__);    \
  } while (0)

#define MMF_CUDA(call)                                                                       \
  do {                                                                                       \
    cudaError_t e_ = (call);                                                                 \
    if (e_ != cudaSuccess) return fail(MMF_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

#define MMF_TRY(expr)                \
  do {                               \
    mmf_status s_ = (expr);          \
    if (s_ != MMF_OK) return s_;     \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool valid_dtype(mmf_dtype d) { return d == MMF_F32 || d == MMF_BF16; }
inline size_t dsize(mmf_dtype d) { return d == MMF_F32 ? 4 : 2; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int32_t row_words(int32_t k) { return 4 * ((k + 63) / 64); }
inline int64_t row_q(int32_t k) { return 16 * (int64_t)row_words(k); }  // int8 codes per row

// ---------------------------------------------------------------------------------------------
// per-device state
// ---------------------------------------------------------------------------------------------
struct DevInfo {
  bool init = false;
  unsigned long long ctx_id = 0;  // the context the kernel attributes below were set in
  int sms = 0;
  int major = 0, minor = 0;
  bool tc_ready = false;
};
DevInfo g_dev[64];
std::mutex g_dev_mu;

// Unique id of the calling thread's current CUDA context (never reused within a process), or 0
// when the driver cannot tell. A device reset ends the context, so per-context state (kernel
// attributes, symbol addresses) is set up again when this id changes.
typedef CUresult (*PfnCtxGetCurrent)(CUcontext*);
typedef CUresult (*PfnCtxGetId)(CUcontext, unsigned long long*);
unsigned long long current_ctx_id() {
  static PfnCtxGetCurrent get_current = nullptr;
  static PfnCtxGetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PfnCtxGetCurrent>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PfnCtxGetId>(fn);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

template <mmf_dtype ZT, mmf_dtype HT>
cudaError_t scan_tile_attrs() {
  cudaError_t e = cudaSuccess;
  const int smem = scan_tile_bytes<ZT>();
  auto set = [&](const void* f) {
    if (e == cudaSuccess) e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  };
  set((const void*)scan_tile_kernel<ZT, HT, false, 0>);
  set((const void*)scan_tile_kernel<ZT, HT, false, 1>);
  set((const void*)scan_tile_kernel<ZT, HT, false, 2>);
  set((const void*)scan_tile_kernel<ZT, HT, true, 0>);
  set((const void*)scan_tile_kernel<ZT, HT, true, 1>);
  set((const void*)scan_tile_kernel<ZT, HT, true, 2>);
  return e;
}

template <mmf_dtype XT, mmf_dtype TT>
cudaError_t head_attrs() {
  const int smem = 200 * 1024;
  cudaError_t e = cudaFuncSetAttribute(head::head_logits_kernel<XT, TT, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(head::head_logits_kernel<XT, TT, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(head::head_logits_kernel<XT, TT, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(head::head_logits_kernel<XT, TT, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return e;
}
cudaError_t head_tc_attrs() {
  return cudaFuncSetAttribute(head::head_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              head::tc_smem_bytes(head::kTcRowsMax));
}


PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

mmf_status device_info(DevInfo** out) {
  int dev = 0;
  MMF_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(MMF_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  const unsigned long long ctx = current_ctx_id();
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& di = g_dev[dev];
  if (di.init && ctx != 0) {
    if (di.ctx_id == 0) di.ctx_id = ctx;          // set up before the context was current
    else if (ctx != di.ctx_id) di = DevInfo();    // a new context (after a reset): set up again
  }
  if (!di.init) {
    di.ctx_id = ctx;
    MMF_CUDA(cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev));
    MMF_CUDA(cudaDeviceGetAttribute(&di.major, cudaDevAttrComputeCapabilityMajor, dev));
    MMF_CUDA(cudaDeviceGetAttribute(&di.minor, cudaDevAttrComputeCapabilityMinor, dev));
    if (di.major == 10 && di.minor == 0) {
      MMF_CUDA(cudaFuncSetAttribute(tc::ternary_gemm_tc_kernel<MMF_F32>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES));
      MMF_CUDA(cudaFuncSetAttribute(tc::ternary_gemm_tc_kernel<MMF_BF16>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES));
      MMF_CUDA(cudaFuncSetAttribute(simt_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    200 * 1024));
      MMF_CUDA(cudaFuncSetAttribute(dec::dec_proj_kernel<MMF_F32, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kMaxSmem));
      MMF_CUDA(cudaFuncSetAttribute(dec::dec_proj_kernel<MMF_F32, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kMaxSmem));
      MMF_CUDA(cudaFuncSetAttribute(dec::dec_proj_kernel<MMF_BF16, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kMaxSmem));
      MMF_CUDA(cudaFuncSetAttribute(dec::dec_proj_kernel<MMF_BF16, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kMaxSmem));
      MMF_CUDA(cudaFuncSetAttribute(dec::dec_proj_kernel<MMF_F32, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kMaxSmem));
      MMF_CUDA(cudaFuncSetAttribute(dec::dec_proj_kernel<MMF_F32, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kMaxSmem));
      MMF_CUDA(cudaFuncSetAttribute(dec::dec_proj_kernel<MMF_BF16, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kMaxSmem));
      MMF_CUDA(cudaFuncSetAttribute(dec::dec_proj_kernel<MMF_BF16, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kMaxSmem));
      MMF_CUDA(cudaFuncSetAttribute(norm_quant_kernel<kRowPlain>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024));
      MMF_CUDA(cudaFuncSetAttribute(norm_quant_kernel<kRowGlu>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024));
      MMF_CUDA(cudaFuncSetAttribute(norm_quant_kernel<kRowGnorm>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024));
      MMF_CUDA((scan_tile_attrs<MMF_F32, MMF_F32>()));
      MMF_CUDA((scan_tile_attrs<MMF_F32, MMF_BF16>()));
      MMF_CUDA((scan_tile_attrs<MMF_BF16, MMF_F32>()));
      MMF_CUDA((scan_tile_attrs<MMF_BF16, MMF_BF16>()));
      MMF_CUDA((head_attrs<MMF_F32, MMF_F32>()));
      MMF_CUDA((head_attrs<MMF_F32, MMF_BF16>()));
      MMF_CUDA((head_attrs<MMF_BF16, MMF_F32>()));
      MMF_CUDA((head_attrs<MMF_BF16, MMF_BF16>()));
      MMF_CUDA(head_tc_attrs());
      MMF_CUDA(cudaFuncSetAttribute(gb::bf16_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, gb::SMEM_BYTES));
      MMF_CUDA(cudaFuncSetAttribute(drow::row_stage_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)(3 * drow::kMaxK * sizeof(float))));
      MMF_CUDA(cudaFuncSetAttribute(sk::ternary_gemm_skinny_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    sk::Layout<16>::SMEM));
      MMF_CUDA(cudaFuncSetAttribute(sk::ternary_gemm_skinny_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    sk::Layout<32>::SMEM));
      MMF_CUDA(cudaFuncSetAttribute(sk::ternary_gemm_skinny_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    sk::Layout<64>::SMEM));
      di.tc_ready = true;
    }
    di.init = true;
  }
  if (!di.tc_ready)
    return fail(MMF_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library runs on sm_100a (B200) only",
                dev, di.major, di.minor);
  *out = &di;
  return MMF_OK;
}

mmf_status get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return fail(MMF_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  return MMF_OK;
}

mmf_status encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t dim0,
                     uint64_t dim1, uint64_t stride1_bytes, uint32_t box0, uint32_t box1,
                     CUtensorMapSwizzle swz) {
  MMF_TRY(get_encoder());
  cuuint64_t dims[2] = {dim0, dim1};
  cuuint64_t strides[1] = {stride1_bytes};
  cuuint32_t box[2] = {box0, box1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MMF_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MMF_OK;
}

// Launches a kernel (cudaLaunchKernelEx; errors surface through check_launch).
template <typename... KArgs, typename... Args>
void launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

mmf_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(e));
  return MMF_OK;
}

// ---------------------------------------------------------------------------------------------
// instrumentation: launch counter and optional per-class event timing
// ---------------------------------------------------------------------------------------------
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_timing{0};
struct TimedRec {
  int cls;
  cudaEvent_t a, b;
  double work;
};
std::mutex g_tmu;
std::vector<TimedRec> g_recs;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t pooled_event() {
  cudaEvent_t e = nullptr;
  if (!g_event_pool.empty()) {
    e = g_event_pool.back();
    g_event_pool.pop_back();
  } else if (cudaEventCreate(&e) != cudaSuccess) {
    e = nullptr;
  }
  return e;
}

// Counts one launch and, when timing is on, brackets it with events on its stream.
struct LaunchScope {
  bool on = false;
  TimedRec rec{};
  cudaStream_t st;
  LaunchScope(int cls, double work, cudaStream_t s) : st(s) {
    g_launches.fetch_add(1);
    if (g_timing.load()) {
      std::lock_guard<std::mutex> lk(g_tmu);
      rec.cls = cls;
      rec.work = work;
      rec.a = pooled_event();
      rec.b = pooled_event();
      on = rec.a && rec.b;
    }
    if (on) cudaEventRecord(rec.a, st);
  }
  ~LaunchScope() {
    if (!on) return;
    cudaEventRecord(rec.b, st);
    std::lock_guard<std::mutex> lk(g_tmu);
    g_recs.push_back(rec);
  }
};

// ---------------------------------------------------------------------------------------------
// internal launchers
// ---------------------------------------------------------------------------------------------
template <mmf_dtype XT, int MODE, int NG>
void nq_vec_launch(const NormQuantArgs& a, int w, int nch, cudaStream_t st) {
  const int64_t rows_per_cta = (kNqThreads / 32) / w;
  const int64_t blocks = (a.m + rows_per_cta - 1) / rows_per_cta;
  int sms = 148;
  {
    DevInfo* di = nullptr;
    if (device_info(&di) == MMF_OK) sms = di->sms;
  }
  // persistent CTAs: as many as are resident at once (occupancy of this instantiation), each
  // walking row blocks gridDim.x apart
  const auto grid_for = [&](const void* fn) {
    static std::mutex mu;
    static std::map<const void*, int> per_sm;
    int n = 0;
    {
      std::lock_guard<std::mutex> lk(mu);
      auto it = per_sm.find(fn);
      if (it == per_sm.end()) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kNqThreads, 0) != cudaSuccess || n < 1) n = 1;
        per_sm[fn] = n;
      } else {
        n = it->second;
      }
    }
    return dim3((unsigned)std::min<int64_t>(blocks, (int64_t)sms * n));
  };
#define MMF_NQ(W_, C_)                                                                    \
  launch_k(norm_quant_vec_kernel<XT, MODE, W_, C_, NG>,                                   \
           grid_for((const void*)norm_quant_vec_kernel<XT, MODE, W_, C_, NG>), dim3(kNqThreads), 0, st, a)
#define MMF_NQ_W(W_) \
  do {                                                                                    \
    if (nch <= 1) MMF_NQ(W_, 1);                                                          \
    else if (nch <= 2) MMF_NQ(W_, 2);                                                     \
    else if (nch <= 3) MMF_NQ(W_, 3);                                                     \
    else if (nch <= 4) MMF_NQ(W_, 4);                                                     \
    else if (nch <= 6) MMF_NQ(W_, 6);                                                     \
    else MMF_NQ(W_, 8);                                                                   \
  } while (0)
  if (w == 1) MMF_NQ_W(1);
  else if (w == 2) MMF_NQ_W(2);
  else MMF_NQ_W(4);
#undef MMF_NQ_W
#undef MMF_NQ
}

template <mmf_dtype XT>
void nq_vec_dispatch(const NormQuantArgs& a, int mode, int w, int nch, cudaStream_t st) {
  if (mode == kRowPlain) {
    if (a.ngain == 1) nq_vec_launch<XT, kRowPlain, 1>(a, w, nch, st);
    else nq_vec_launch<XT, kRowPlain, 3>(a, w, nch, st);
  } else if (mode == kRowGlu) {
    nq_vec_launch<XT, kRowGlu, 1>(a, w, nch, st);
  } else {
    nq_vec_launch<XT, kRowGnorm, 1>(a, w, nch, st);
  }
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mmf_status launch_norm_quant(const NormQuantArgs& a, int mode, cudaStream_t st) {
  if (a.m == 0) return MMF_OK;
  const double es = a.xdt == MMF_F32 ? 4.0 : 2.0;
  double in_row = (mode == kRowGlu ? 2.0 : 1.0) * a.k * es;
  if (mode == kRowGnorm) in_row += a.k * (a.gdt == MMF_F32 ? 4.0 : 2.0);
  LaunchScope ls(MMF_KERNEL_NORM_QUANT, (double)a.m * (in_row + a.ngain * ((double)a.ldq + 4.0)), st);
  // row-group-in-registers variant when sizes and alignment allow it
  const size_t xes = dsize(a.xdt);
  bool vec = a.k % 8 == 0 && a.k <= 8 * 32 * 4 * 8 && al16(a.x) && (a.ldx * xes) % 16 == 0 &&
             (mode == kRowPlain || a.ngain == 1);
  if (mode == kRowGnorm)
    vec = vec && a.gdt == a.xdt && al16(a.g) && (a.ldg * xes) % 16 == 0 && al16(a.gw);
  for (int j = 0; j < a.ngain; ++j) vec = vec && al16(a.gain[j]) && al16(a.q[j]);
  if (vec) {
    // smallest row group (1, 2 or 4 warps) whose threads hold at most `cap` 8-value chunks: the
    // row, its prefetched successor and the register-resident gains of those columns then fit
    // in about 100 registers (more warps per row only when the row needs it)
    const int nck = a.k / 8;
    const int cap = (mode == kRowPlain && a.ngain == 1) ? 4 : 2;
    int w = 1;
    while (w < 4 && (nck + 32 * w - 1) / (32 * w) > cap) w *= 2;
    const int nch = (nck + 32 * w - 1) / (32 * w);
    if (a.xdt == MMF_F32) nq_vec_dispatch<MMF_F32>(a, mode, w, nch, st);
    else nq_vec_dispatch<MMF_BF16>(a, mode, w, nch, st);
    return check_launch("norm_quant_vec_kernel");
  }
  const size_t smem = (size_t)a.k * sizeof(float);
  const int threads = a.k >= 2048 ? 256 : 128;
  dim3 grid((unsigned)a.m);
  if (mode == kRowPlain) launch_k(norm_quant_kernel<kRowPlain>, grid, dim3(threads), smem, st, a);
  else if (mode == kRowGlu) launch_k(norm_quant_kernel<kRowGlu>, grid, dim3(threads), smem, st, a);
  else launch_k(norm_quant_kernel<kRowGnorm>, grid, dim3(threads), smem, st, a);
  return check_launch("norm_quant_kernel");
}

bool use_tensor_path(int64_t m) {
  const int p = g_gemm_path.load();
  if (p == MMF_GEMM_TENSOR) return true;
  if (p == MMF_GEMM_SIMT) return false;
  return m >= kSimtMT;  // 8 rows and up: the tensor-core kernel's cost barely depends on m
}

// gate_proj forms the GLU product in its epilogue when the tensor engine runs it and the inner
// size splits into 64-row gate/up tile halves.
bool glu_fused(int64_t m, int32_t inner) { return use_tensor_path(m) && inner % tc::GLU_ROWS == 0; }

mmf_status launch_gemm(const GemmArgs& g, const DevInfo& di, cudaStream_t st) {
  if (g.m == 0) return MMF_OK;
  if (!use_tensor_path(g.m)) {
    int maxn = 0;
    for (int s = 0; s < g.nseg; ++s) maxn = std::max(maxn, g.seg[s].n);
    for (int s = 0; s < g.nseg; ++s)
      if (g.seg[s].glu) return fail(MMF_ERR_UNSUPPORTED, "GLU segments run on the tensor engine only");
    const int nchunk = g.kw / 4;
    const size_t smem = (size_t)kSimtMT * nchunk * 4 * sizeof(uint4);
    if (smem > 200 * 1024) return fail(MMF_ERR_UNSUPPORTED, "K=%d too large for the CUDA-core engine", g.k);
    const int gx = std::min((maxn + 31) / 32, di.sms * 8);
    dim3 grid((unsigned)std::max(gx, 1), (unsigned)((g.m + kSimtMT - 1) / kSimtMT), (unsigned)g.nseg);
    double bytes = 0;
    const double yes = g.ydt == MMF_F32 ? 4.0 : 2.0;
    for (int s = 0; s < g.nseg; ++s)
      bytes += (double)g.seg[s].n * g.kw * 4.0 + (double)g.m * g.ldq + (double)g.m * g.seg[s].n * yes *
               (g.seg[s].res ? 2.0 : 1.0);
    LaunchScope ls(MMF_KERNEL_GEMM_SIMT, bytes, st);
    launch_k(simt_gemm_kernel, grid, dim3(256), smem, st, g);
    return check_launch("simt_gemm_kernel");
  }
  tc::Params P;
  memset(&P, 0, sizeof(P));
  P.g = g;
  P.m_tiles = (int32_t)((g.m + tc::BN - 1) / tc::BN);
  int32_t tiles = 0;
  for (int s = 0; s < g.nseg; ++s) {
    const GemmSeg& S = g.seg[s];
    if (S.glu && (S.glu_inner % tc::GLU_ROWS != 0 || S.n != 2 * S.glu_inner || S.acc != nullptr || S.res != nullptr))
      return fail(MMF_ERR_INVALID_ARG, "GLU segment needs inner %% 64 == 0, n == 2 * inner, no taps, no residual");
    P.tile_start[s] = tiles;
    tiles += (S.glu ? S.glu_inner / tc::GLU_ROWS : (S.n + tc::BM - 1) / tc::BM) * P.m_tiles;
    MMF_TRY(encode_2d(&P.act_map[s], CU_TENSOR_MAP_DATA_TYPE_UINT8, S.q, (uint64_t)g.ldq,
                      (uint64_t)g.m, (uint64_t)g.ldq, tc::ACT_BOX, tc::BN, CU_TENSOR_MAP_SWIZZLE_128B));
    MMF_TRY(encode_2d(&P.w_map[s], CU_TENSOR_MAP_DATA_TYPE_UINT32, S.codes, (uint64_t)g.kw,
                      (uint64_t)S.n, (uint64_t)g.kw * 4, tc::W_WORDS_PER_ROW,
                      S.glu ? tc::GLU_ROWS : tc::BM, CU_TENSOR_MAP_SWIZZLE_64B));
  }
  P.tile_start[g.nseg] = tiles;
  P.num_kb = (int32_t)((g.ldq + tc::BK - 1) / tc::BK);
  P.small_acc = (int64_t)127 * g.k < ((int64_t)1 << 22) ? 1 : 0;
  P.wait_limit_us = g_wait_limit.load();
  const int grid = std::min(tiles, di.sms);
  double ops = 0;
  for (int s = 0; s < g.nseg; ++s) ops += 2.0 * (double)g.m * g.seg[s].n * g.k;
  LaunchScope ls(MMF_KERNEL_GEMM_TC, ops, st);
  if (g.ydt == MMF_F32)
    launch_k(tc::ternary_gemm_tc_kernel<MMF_F32>, dim3(grid), dim3(tc::NUM_THREADS), tc::SMEM_BYTES, st, P);
  else
    launch_k(tc::ternary_gemm_tc_kernel<MMF_BF16>, dim3(grid), dim3(tc::NUM_THREADS), tc::SMEM_BYTES, st, P);
  return check_launch("ternary_gemm_tc_kernel");
}

// Steps per chunk of the chunked scan: 16 (one register prefetch block per thread) up to 2048
// steps, then a multiple of 16 giving at most 128 chunks.
inline int32_t scan_chunk(int64_t t) {
  if (t <= 2048) return 16;
  const int64_t c = (t + 127) / 128;
  return (int32_t)((c + 15) / 16 * 16);
}
// Steps per chunk of the shared-memory staged scan: 64 (four double-buffered tiles) up to 8192
// steps, then a multiple of 16 giving at most 128 chunks.
inline int32_t scan_tile_chunk(int64_t t) {
  if (t <= 8192) return 64;
  const int64_t c = (t + 127) / 128;
  return (int32_t)((c + 15) / 16 * 16);
}
// Scratch of the chunked scan for m = b*t tokens of d channels: three [b][nchunk][d] float
// arrays. b * nchunk <= ceil(m / 8) whenever t > 16 (shorter sequences need no scratch):
// chunks are at least 16 steps, so nchunk = ceil(t/16) <= t/8, and past 2048 (register path) or
// 8192 (staged path) steps nchunk <= 128 < t/16.
inline size_t scan_ws_bytes(int64_t m, int32_t d) {
  return 3 * align256((size_t)d * 4 * (size_t)((m + 7) / 8));
}

template <mmf_dtype ZT, mmf_dtype HT, int VEC, bool GATED>
void scan_launch_gated(const ScanArgs& a, cudaStream_t st) {
  const unsigned gx = (unsigned)((a.d / VEC + kScanThreads - 1) / kScanThreads);
  if (a.nchunk == 1) {
    launch_k(scan_apply_kernel<ZT, HT, VEC, true, GATED>, dim3(gx, 1, a.b), dim3(kScanThreads), 0, st, a);
    return;
  }
  launch_k(scan_aggregate_kernel<ZT, VEC, GATED>, dim3(gx, a.nchunk, a.b), dim3(kScanThreads), 0, st, a);
  launch_k(scan_carry_kernel, dim3((unsigned)((a.d + kScanThreads - 1) / kScanThreads), a.b), dim3(kScanThreads), 0, st, a);
  launch_k(scan_apply_kernel<ZT, HT, VEC, false, GATED>, dim3(gx, a.nchunk, a.b), dim3(kScanThreads), 0, st, a);
}

template <mmf_dtype ZT, mmf_dtype HT, int VEC>
void scan_launch_typed(const ScanArgs& a, cudaStream_t st) {
  if (a.gated) scan_launch_gated<ZT, HT, VEC, true>(a, st);
  else scan_launch_gated<ZT, HT, VEC, false>(a, st);
}

// Tiled (shared-memory staged) phases; needs 16-byte aligned rows and an even channel count.
template <mmf_dtype ZT, mmf_dtype HT, bool GATED>
void scan_tiled_gated(const ScanArgs& a, cudaStream_t st) {
  constexpr int smem = scan_tile_bytes<ZT>();
  const unsigned gx = (unsigned)((a.d + kScanTileCh - 1) / kScanTileCh);
  if (a.nchunk == 1) {
    launch_k(scan_tile_kernel<ZT, HT, GATED, 2>, dim3(gx, 1, a.b), dim3(kScanThreads), smem, st, a);
    return;
  }
  launch_k(scan_tile_kernel<ZT, HT, GATED, 0>, dim3(gx, a.nchunk, a.b), dim3(kScanThreads), smem, st, a);
  launch_k(scan_carry_kernel, dim3((unsigned)((a.d + kScanThreads - 1) / kScanThreads), a.b), dim3(kScanThreads), 0, st, a);
  launch_k(scan_tile_kernel<ZT, HT, GATED, 1>, dim3(gx, a.nchunk, a.b), dim3(kScanThreads), smem, st, a);
}
template <mmf_dtype ZT, mmf_dtype HT>
void scan_tiled_typed(const ScanArgs& a, cudaStream_t st) {
  if (a.gated) scan_tiled_gated<ZT, HT, true>(a, st);
  else scan_tiled_gated<ZT, HT, false>(a, st);
}

template <int VEC>
void scan_launch_vec(const ScanArgs& a, cudaStream_t st) {
  if (a.zdt == MMF_F32 && a.hdt == MMF_F32) scan_launch_typed<MMF_F32, MMF_F32, VEC>(a, st);
  else if (a.zdt == MMF_F32) scan_launch_typed<MMF_F32, MMF_BF16, VEC>(a, st);
  else if (a.hdt == MMF_F32) scan_launch_typed<MMF_BF16, MMF_F32, VEC>(a, st);
  else scan_launch_typed<MMF_BF16, MMF_BF16, VEC>(a, st);
}

// ws: scan_ws_bytes(b*t, d) bytes (unused when t <= 16, or while the sequence is one chunk).
mmf_status launch_scan(ScanArgs a, void* ws, cudaStream_t st) {
  if ((int64_t)a.b * a.d == 0) return MMF_OK;
  const int64_t chans = (int64_t)a.b * a.d;
  if (a.t == 0) {
    // no steps: the final state is the initial one
    if (a.h_last) {
      if (a.h0) {
        cudaError_t e = cudaMemcpyAsync(a.h_last, a.h0, chans * sizeof(float), cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "cudaMemcpyAsync: %s", cudaGetErrorString(e));
      } else {
        cudaError_t e = cudaMemsetAsync(a.h_last, 0, chans * sizeof(float), st);
        if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
      }
    }
    return MMF_OK;
  }
  const size_t zes = dsize(a.zdt), hes = dsize(a.hdt);
  const auto aligned = [](const void* q, size_t n) { return (reinterpret_cast<uintptr_t>(q) % n) == 0; };
  const bool pair = (a.d % 2 == 0) && (a.zstride % 2 == 0) && aligned(a.zf, 2 * zes) && aligned(a.zi, 2 * zes) &&
                    aligned(a.h, 2 * hes);
  const bool tiled = pair && (a.zstride * zes) % 16 == 0 && (a.d * zes) % 16 == 0 && aligned(a.zf, 16) &&
                     aligned(a.zi, 16) && aligned(a.h0, 8) && aligned(a.h_last, 8);
  const int32_t chunk = tiled ? scan_tile_chunk(a.t) : (a.t <= 16 ? (int32_t)a.t : scan_chunk(a.t));
  if (a.t <= chunk) {
    a.chunk = (int32_t)a.t;
    a.nchunk = 1;
  } else {
    a.chunk = chunk;
    a.nchunk = (int32_t)((a.t + a.chunk - 1) / a.chunk);
    const size_t arr = align256((size_t)a.d * 4 * (size_t)(((int64_t)a.b * a.t + 7) / 8));
    uint8_t* p = reinterpret_cast<uint8_t*>(ws);
    a.agg_a = reinterpret_cast<float*>(p);
    a.agg_b = reinterpret_cast<float*>(p + arr);
    a.cin = reinterpret_cast<float*>(p + 2 * arr);
  }
  const double zb = (double)zes, hb = (double)hes;
  LaunchScope ls(MMF_KERNEL_SCAN, (double)chans * a.t * (2.0 * zb + hb) + (double)chans * 4.0 *
                 ((a.h0 ? 1.0 : 0.0) + (a.h_last ? 1.0 : 0.0)), st);
  if (a.nchunk > 1) g_launches.fetch_add(2);  // three kernels under one timing scope
  if (tiled) {
    if (a.zdt == MMF_F32 && a.hdt == MMF_F32) scan_tiled_typed<MMF_F32, MMF_F32>(a, st);
    else if (a.zdt == MMF_F32) scan_tiled_typed<MMF_F32, MMF_BF16>(a, st);
    else if (a.hdt == MMF_F32) scan_tiled_typed<MMF_BF16, MMF_F32>(a, st);
    else scan_tiled_typed<MMF_BF16, MMF_BF16>(a, st);
  } else if (pair) {
    scan_launch_vec<2>(a, st);
  } else {
    scan_launch_vec<1>(a, st);
  }
  return check_launch("hgrn scan kernels");
}

mmf_status check_ternary(const mmf_ternary* w, int32_t n, int32_t k, const char* name) {
  MMF_CHECK_ARG(w != nullptr, "%s: null weight descriptor", name);
  MMF_CHECK_ARG(w->codes && w->scale, "%s: null codes or scale", name);
  MMF_CHECK_ARG(aligned16(w->codes), "%s: codes not 16-byte aligned", name);
  MMF_CHECK_ARG(w->n == n && w->k == k, "%s: shape [%d][%d], expected [%d][%d]", name, w->n, w->k, n, k);
  return MMF_OK;
}

// Workspace carve-up of one block forward over m tokens.
struct BlockWs {
  int8_t* q3;  // [3][m][ldq_d]
  float* deq;  // [6][m]
  void* z;     // [3][m][d]: the i, f, g planes
  void* h;     // [m][d]
  int8_t* qo;  // [m][ldq_d]
  void* x1;    // [m][d]
  int8_t* qg;  // [m][ldq_d]
  void* gu;    // [m][2I]
  int8_t* qd;  // [m][ldq_I]
  void* scan;  // chunked-scan scratch
  size_t bytes;
};

BlockWs block_ws(void* base, int64_t m, int32_t d, int32_t inner, mmf_dtype dt) {
  BlockWs w;
  uint8_t* p = reinterpret_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* r = p ? p + off : nullptr;
    off += align256(bytes);
    return r;
  };
  const size_t es = dsize(dt);
  w.q3 = reinterpret_cast<int8_t*>(take(3 * m * row_q(d)));
  w.deq = reinterpret_cast<float*>(take(6 * m * sizeof(float)));
  w.z = take(m * 3 * (size_t)d * es);
  w.h = take(m * (size_t)d * es);
  w.qo = reinterpret_cast<int8_t*>(take(m * row_q(d)));
  w.x1 = take(m * (size_t)d * es);
  w.qg = reinterpret_cast<int8_t*>(take(m * row_q(d)));
  w.gu = take(m * 2 * (size_t)inner * es);
  w.qd = reinterpret_cast<int8_t*>(take(m * row_q(inner)));
  w.scan = take(scan_ws_bytes(m, d));
  w.bytes = off;
  return w;
}

GemmSeg make_seg(const int8_t* q, const float* deq, const mmf_ternary& w, void* y, int64_t ldy,
                 int32_t ycol, const void* res, int64_t ldres, int32_t* acc, int64_t ldacc) {
  GemmSeg s;
  memset(&s, 0, sizeof(s));
  s.q = q;
  s.deq = deq;
  s.codes = w.codes;
  s.sw = w.scale;
  s.n = w.n;
  s.y = y;
  s.ldy = ldy;
  s.ycol = ycol;
  s.res = res;
  s.ldres = ldres;
  s.rescol = 0;
  s.acc = acc;
  s.ldacc = ldacc;
  return s;
}

mmf_status check_block(const mmf_block_weights* w) {
  MMF_CHECK_ARG(w != nullptr, "null block weights");
  MMF_CHECK_ARG(w->d > 0 && w->inner > 0, "bad block sizes d=%d inner=%d", w->d, w->inner);
  MMF_CHECK_ARG(w->d <= 32768 && w->inner <= 32768, "block sizes above 32768 are not supported");
  MMF_CHECK_ARG(w->eps >= 0.0f, "negative eps");
  MMF_TRY(check_ternary(&w->i, w->d, w->d, "i_proj"));
  MMF_TRY(check_ternary(&w->f, w->d, w->d, "f_proj"));
  MMF_TRY(check_ternary(&w->g, w->d, w->d, "g_proj"));
  MMF_TRY(check_ternary(&w->o, w->d, w->d, "o_proj"));
  MMF_TRY(check_ternary(&w->gate, 2 * w->inner, w->d, "gate_proj"));
  MMF_TRY(check_ternary(&w->down, w->d, w->inner, "down_proj"));
  return MMF_OK;
}

// The block forward on m = b*t tokens; ws already validated.
mmf_status run_block(const mmf_block_weights* w, const void* x, mmf_dtype dt, int32_t b, int64_t t,
                     const float* h0, void* y, float* h_last, const BlockWs& W, const DevInfo& di,
                     cudaStream_t st) {
  const int64_t m = (int64_t)b * t;
  const int32_t d = w->d, inner = w->inner;
  const int64_t ldq_d = row_q(d), ldq_i = row_q(inner);
  const size_t es = dsize(dt);
  float* deq = W.deq;
  // 1. RMSNorm + int8 quant of x with the three gains of i/f/g_proj (one shared rms)
  NormQuantArgs nq;
  memset(&nq, 0, sizeof(nq));
  nq.x = x; nq.ldx = d; nq.xdt = dt; nq.m = m; nq.k = d; nq.eps = w->eps; nq.ngain = 3;
  nq.gain[0] = w->nw_i; nq.gain[1] = w->nw_f; nq.gain[2] = w->nw_g;
  for (int j = 0; j < 3; ++j) {
    nq.q[j] = W.q3 + j * m * ldq_d;
    nq.deq[j] = deq + j * m;
  }
  nq.ldq = ldq_d;
  MMF_TRY(launch_norm_quant(nq, kRowPlain, st));
  // 2. i/f/g projections in one grouped GEMM: z = [zi | zf | g]
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.m = m; g.k = d; g.kw = row_words(d); g.ldq = ldq_d; g.ydt = dt; g.nseg = 3;
  // z is three planes [i | f | g] of [m][d], so the scan and g_norm read contiguous rows
  uint8_t* zp = reinterpret_cast<uint8_t*>(W.z);
  const size_t plane = (size_t)m * d * es;
  g.seg[0] = make_seg(W.q3, deq, w->i, zp, d, 0, nullptr, 0, nullptr, 0);
  g.seg[1] = make_seg(W.q3 + m * ldq_d, deq + m, w->f, zp + plane, d, 0, nullptr, 0, nullptr, 0);
  g.seg[2] = make_seg(W.q3 + 2 * m * ldq_d, deq + 2 * m, w->g, zp + 2 * plane, d, 0, nullptr, 0, nullptr, 0);
  MMF_TRY(launch_gemm(g, di, st));
  // 3. HGRN scan with gates
  ScanArgs sa;
  memset(&sa, 0, sizeof(sa));
  sa.zf = zp + plane;
  sa.zi = zp;
  sa.zdt = dt; sa.zstride = d; sa.b = b; sa.t = t; sa.d = d;
  sa.h0 = h0; sa.h = W.h; sa.hdt = dt; sa.h_last = h_last;
  MMF_TRY(launch_scan(sa, W.scan, st));
  // 4. g_norm (RMSNorm(h) * gnorm_w * SiLU(g)) fused with o_proj's RMSNorm + quant
  memset(&nq, 0, sizeof(nq));
  nq.x = W.h; nq.ldx = d; nq.xdt = dt;
  nq.g = zp + 2 * plane; nq.ldg = d; nq.gdt = dt;
  nq.gw = w->gnorm_w; nq.m = m; nq.k = d; nq.eps = w->eps; nq.ngain = 1; nq.gain[0] = w->nw_o;
  nq.q[0] = W.qo; nq.deq[0] = deq + 3 * m; nq.ldq = ldq_d;
  MMF_TRY(launch_norm_quant(nq, kRowGnorm, st));
  // 5. o_proj + residual: x1 = x + o_proj(u)
  memset(&g, 0, sizeof(g));
  g.m = m; g.k = d; g.kw = row_words(d); g.ldq = ldq_d; g.ydt = dt; g.nseg = 1;
  g.seg[0] = make_seg(W.qo, deq + 3 * m, w->o, W.x1, d, 0, x, d, nullptr, 0);
  MMF_TRY(launch_gemm(g, di, st));
  // 6. gate_proj input norm + quant
  memset(&nq, 0, sizeof(nq));
  nq.x = W.x1; nq.ldx = d; nq.xdt = dt; nq.m = m; nq.k = d; nq.eps = w->eps; nq.ngain = 1;
  nq.gain[0] = w->nw_gate; nq.q[0] = W.qg; nq.deq[0] = deq + 4 * m; nq.ldq = ldq_d;
  MMF_TRY(launch_norm_quant(nq, kRowPlain, st));
  // 7. gate_proj. The tensor engine pairs gate and up rows in one tile and writes
  //    v = SiLU(gate) * up directly ([m][inner] in the gu buffer); otherwise gu = [gate | up].
  const bool fuse_glu = glu_fused(m, inner);
  memset(&g, 0, sizeof(g));
  g.m = m; g.k = d; g.kw = row_words(d); g.ldq = ldq_d; g.ydt = dt; g.nseg = 1;
  g.seg[0] = make_seg(W.qg, deq + 4 * m, w->gate, W.gu, fuse_glu ? inner : 2 * inner, 0, nullptr, 0, nullptr, 0);
  if (fuse_glu) {
    g.seg[0].glu = 1;
    g.seg[0].glu_inner = inner;
  }
  MMF_TRY(launch_gemm(g, di, st));
  // 8. down_proj's RMSNorm + quant of v (formed here from [gate | up] when not fused above)
  memset(&nq, 0, sizeof(nq));
  nq.x = W.gu; nq.ldx = fuse_glu ? inner : 2 * inner; nq.xdt = dt; nq.m = m; nq.k = inner; nq.eps = w->eps;
  nq.ngain = 1; nq.gain[0] = w->nw_down; nq.q[0] = W.qd; nq.deq[0] = deq + 5 * m; nq.ldq = ldq_i;
  MMF_TRY(launch_norm_quant(nq, fuse_glu ? kRowPlain : kRowGlu, st));
  // 9. down_proj + residual: y = x1 + down_proj(v)
  memset(&g, 0, sizeof(g));
  g.m = m; g.k = inner; g.kw = row_words(inner); g.ldq = ldq_i; g.ydt = dt; g.nseg = 1;
  g.seg[0] = make_seg(W.qd, deq + 5 * m, w->down, y, d, 0, W.x1, d, nullptr, 0);
  return launch_gemm(g, di, st);
}

// Workspace carve-up of one decode step on the skinny tensor-core path (b <= 64 rows): the
// integer products of the current group, the codes and factors of the four quantisations, x1 and v.
struct SkWs {
  int32_t* acc;  // [b][max(3d, 2I)]
  int8_t* q3;    // [3][b][ldq_d]
  int8_t* qo;    // [b][ldq_d]
  int8_t* qg;    // [b][ldq_d]
  int8_t* qd;    // [b][ldq_I]
  float* deq;    // [6][b]
  void* x1;      // [b][d]
  void* v;       // [b][I]
  size_t bytes;
};
SkWs sk_ws(void* base, int64_t m, int32_t d, int32_t inner) {
  SkWs w;
  uint8_t* p = reinterpret_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* r = p ? p + off : nullptr;
    off += align256(bytes);
    return r;
  };
  w.acc = reinterpret_cast<int32_t*>(take((size_t)m * std::max(3 * d, 2 * inner) * 4));
  w.q3 = reinterpret_cast<int8_t*>(take(3 * m * row_q(d)));
  w.qo = reinterpret_cast<int8_t*>(take(m * row_q(d)));
  w.qg = reinterpret_cast<int8_t*>(take(m * row_q(d)));
  w.qd = reinterpret_cast<int8_t*>(take(m * row_q(inner)));
  w.deq = reinterpret_cast<float*>(take(6 * m * sizeof(float)));
  w.x1 = take((size_t)m * d * 4);
  w.v = take((size_t)m * inner * 4);
  w.bytes = off;
  return w;
}
// Bytes of a decode step's workspace before its two layer-output buffers: the largest of the
// block path's, the skinny path's (the fused path uses a prefix of either).
size_t decode_ws_head(int64_t m, int32_t d, int32_t inner) {
  return std::max(block_ws(nullptr, m, d, inner, MMF_F32).bytes, sk_ws(nullptr, m, d, inner).bytes);
}

struct SkSeg {
  const int8_t* q;        // [m][ldq] codes
  const uint32_t* codes;  // [n][kw] packed weights
  int32_t n;
  int32_t* acc;           // acc[row * ldacc + col]
};

// acc = q . t^T for m <= 64 rows on the skinny tensor-core kernel (one launch, up to three
// segments sharing m, k and the accumulator stride).
mmf_status launch_skinny(const SkSeg* segs, int nseg, int64_t m, int32_t k, int64_t ldq, int64_t ldacc,
                         const DevInfo& di, cudaStream_t st) {
  if (m == 0) return MMF_OK;
  if (m > 64) return fail(MMF_ERR_UNSUPPORTED, "skinny product: %lld rows (at most 64)", (long long)m);
  sk::Params P;
  memset(&P, 0, sizeof(P));
  const int bn = m <= 16 ? 16 : (m <= 32 ? 32 : 64);
  const int32_t kw = row_words(k);
  int32_t tiles = 0;
  for (int s = 0; s < nseg; ++s) {
    P.tile_start[s] = tiles;
    tiles += (segs[s].n + sk::BM - 1) / sk::BM;
    MMF_TRY(encode_2d(&P.act_map[s], CU_TENSOR_MAP_DATA_TYPE_UINT8, segs[s].q, (uint64_t)ldq, (uint64_t)m,
                      (uint64_t)ldq, 128, (uint32_t)bn, CU_TENSOR_MAP_SWIZZLE_128B));
    MMF_TRY(encode_2d(&P.w_map[s], CU_TENSOR_MAP_DATA_TYPE_UINT32, segs[s].codes, (uint64_t)kw, (uint64_t)segs[s].n,
                      (uint64_t)kw * 4, sk::W_WORDS_PER_ROW, sk::BM, CU_TENSOR_MAP_SWIZZLE_64B));
    P.acc[s] = segs[s].acc;
    P.n[s] = segs[s].n;
  }
  P.tile_start[nseg] = tiles;
  P.nseg = nseg;
  P.m = (int32_t)m;
  P.ldacc = ldacc;
  P.num_kb = (int32_t)((ldq + sk::BK - 1) / sk::BK);
  // the largest power-of-two split (<= 8) that keeps one CTA per SM and at least one k-block each
  int splits = 1;
  while (splits * 2 <= sk::MAX_SPLITS && tiles * splits * 2 <= di.sms && splits * 2 <= P.num_kb) splits *= 2;
  P.splits = splits;
  P.kb_per_split = (P.num_kb + splits - 1) / splits;
  P.wait_limit_us = g_wait_limit.load();
  double ops = 0;
  for (int s = 0; s < nseg; ++s) ops += 2.0 * (double)m * segs[s].n * k;
  LaunchScope ls(MMF_KERNEL_GEMM_TC, ops, st);
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)(tiles * splits));
  cfg.blockDim = dim3(sk::NUM_THREADS);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)splits;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = splits > 1 ? 2 : 1;
  if (bn == 16) {
    cfg.dynamicSmemBytes = sk::Layout<16>::SMEM;
    cudaLaunchKernelEx(&cfg, sk::ternary_gemm_skinny_kernel<16>, P);
  } else if (bn == 32) {
    cfg.dynamicSmemBytes = sk::Layout<32>::SMEM;
    cudaLaunchKernelEx(&cfg, sk::ternary_gemm_skinny_kernel<32>, P);
  } else {
    cfg.dynamicSmemBytes = sk::Layout<64>::SMEM;
    cudaLaunchKernelEx(&cfg, sk::ternary_gemm_skinny_kernel<64>, P);
  }
  return check_launch("ternary_gemm_skinny_kernel");
}

mmf_status launch_row_stage(const drow::Args& a, int64_t b, cudaStream_t st) {
  const int kv = (a.mode == drow::kGate) ? a.inner : a.d;
  const double es = a.dt == MMF_F32 ? 4.0 : 2.0;
  LaunchScope ls(MMF_KERNEL_NORM_QUANT, (double)b * kv * (es + 4.0 + a.ngain), st);
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)b);
  cfg.blockDim = dim3(drow::kThreads);
  cfg.dynamicSmemBytes = drow::row_stage_smem(a.mode, a.d, a.inner, a.ngain);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, drow::row_stage_kernel, a);
  return check_launch("row_stage_kernel");
}

mmf_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return MMF_OK;
  if (ws == nullptr || ws_bytes < need)
    return fail(MMF_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", ws ? ws_bytes : (size_t)0, need);
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(MMF_ERR_WORKSPACE, "workspace not 256-byte aligned");
  return MMF_OK;
}

// ---------------------------------------------------------------------------------------------
// static scratch of the allocation-free BitLinear entry point
// ---------------------------------------------------------------------------------------------
// Device-side storage; in host code `g_noalloc_scratch` only names the symbol, so its device
// address is looked up once per device with cudaGetSymbolAddress and passed to the kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MMF_NOALLOC_SCRATCH_BYTES];
// Looked up once per device and context: a device reset ends the context, and the address is
// looked up again in the next one.
void* g_noalloc_ptr[64] = {};
unsigned long long g_noalloc_ctx[64] = {};
std::mutex g_noalloc_mu;

mmf_status noalloc_scratch(void** out) {
  int dev = 0;
  MMF_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(MMF_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  const unsigned long long ctx = current_ctx_id();
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr || (ctx != 0 && g_noalloc_ctx[dev] != 0 && ctx != g_noalloc_ctx[dev])) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(MMF_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
  } else if (g_noalloc_ctx[dev] == 0) {
    g_noalloc_ctx[dev] = ctx;
  }
  *out = g_noalloc_ptr[dev];
  return MMF_OK;
}

// Scratch of the head: the partial maxima, one (logit, index) per CTA and token row of a pass
// (CUDA-core form: CTAs of at least head::kMinRowsPerCta vocabulary rows, head::kRows rows a pass;
// tensor-core form: CTAs of head::kTcBM rows, head::kTcRowsMax rows a pass), then the bf16 hi / lo
// token rows of a tensor-core pass ([2 * kTcRowsMax][d]).
size_t head_parts_bytes(int32_t vocab) {
  const size_t simt = (size_t)((vocab + head::kMinRowsPerCta - 1) / head::kMinRowsPerCta) * head::kRows;
  const size_t tc = (size_t)((vocab + head::kTcBM - 1) / head::kTcBM) * head::kTcRowsMax;
  return align256(std::max(simt, tc) * 4);
}
size_t head_ws_bytes(int32_t vocab, int32_t d) {
  return 2 * head_parts_bytes(vocab) + align256((size_t)2 * head::kTcRowsMax * std::max(d, 0) * 2);
}

template <mmf_dtype XT, mmf_dtype TT>
void head_launch(head::Args a, int nb, int nparts, int32_t* ids, cudaStream_t st) {
  const size_t smem = (size_t)nb * a.d * 4;
#define MMF_HEAD(NB_) launch_k(head::head_logits_kernel<XT, TT, NB_>, dim3((unsigned)nparts), dim3(head::kThreads), smem, st, a)
  if (nb == 8) MMF_HEAD(8);
  else if (nb == 4) MMF_HEAD(4);
  else if (nb == 2) MMF_HEAD(2);
  else MMF_HEAD(1);
#undef MMF_HEAD
  launch_k(head::head_argmax_kernel, dim3((unsigned)((nb + head::kWarps - 1) / head::kWarps)), dim3(head::kThreads), 0, st,
           (const float*)a.pmax, (const int32_t*)a.pidx, nparts, (int)head::kRows, nb, ids);
}

// One tensor-core pass of nb <= kTcRowsMax token rows: hi / lo rows, logits tiles, argmax.
mmf_status head_tc_pass(const void* x, mmf_dtype xdt, int nb, int d, const float* norm_w, float eps, const void* table,
                        int32_t vocab, float* logits, float* pmax, int32_t* pidx, __nv_bfloat16* xs, int32_t* ids,
                        cudaStream_t st) {
  const int h = (nb + 15) / 16 * 16;
  head::TcParams P;
  memset(&P, 0, sizeof(P));
  MMF_TRY(encode_2d(&P.tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, table, (uint64_t)d, (uint64_t)vocab, (uint64_t)d * 2,
                    head::kTcBK, head::kTcBM, CU_TENSOR_MAP_SWIZZLE_128B));
  MMF_TRY(encode_2d(&P.xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, xs, (uint64_t)d, (uint64_t)(2 * h), (uint64_t)d * 2,
                    head::kTcBK, (uint32_t)(2 * h), CU_TENSOR_MAP_SWIZZLE_128B));
  P.nb = nb; P.h = h;
  P.num_kb = (d + head::kTcBK - 1) / head::kTcBK;
  P.vocab = vocab; P.logits = logits; P.ld_logits = vocab;
  P.pmax = pmax; P.pidx = pidx;
  uint32_t cols = 32;
  while (cols < (uint32_t)(2 * h)) cols <<= 1;
  P.tmem_cols = cols;
  P.wait_limit_us = g_wait_limit.load();
  const int tiles = (vocab + head::kTcBM - 1) / head::kTcBM;
  if (xdt == MMF_F32)
    launch_k(head::head_pack_kernel<MMF_F32>, dim3((unsigned)h), dim3(head::kThreads), 0, st, x, d, norm_w, eps, nb, h, xs);
  else
    launch_k(head::head_pack_kernel<MMF_BF16>, dim3((unsigned)h), dim3(head::kThreads), 0, st, x, d, norm_w, eps, nb, h, xs);
  launch_k(head::head_tc_kernel, dim3((unsigned)tiles), dim3(head::kTcThreads), (size_t)head::tc_smem_bytes(h), st, P);
  launch_k(head::head_argmax_kernel, dim3((unsigned)((nb + head::kWarps - 1) / head::kWarps)), dim3(head::kThreads), 0, st,
           (const float*)pmax, (const int32_t*)pidx, tiles, (int)head::kTcRowsMax, nb, ids);
  return MMF_OK;
}

}  // namespace

// =============================================================================================
// exported C ABI
// =============================================================================================
// Tensor-core form of mmf_bitlinear_backward: the bf16 operand arrays (row pitch rounded up to 8
// elements) and the K split of both products, from (m, k, n) alone so that the workspace query
// and the launch agree. dr's arrays and dW's share the space after rho (the products run in
// turn on one stream).
struct LinBwdPlan {
  int64_t ld_n, ld_m;
  size_t rho, mux, dr_hi, dr_lo, tt, dr_part, dw_hi, dw_lo, qt, dw_part, dnw_part, bytes;
  int dr_split, dr_kbc, dw_split, dw_kbc, dnw_split, dnw_rows;
};
// Splits of K so that an M x N product with few tiles still covers the SMs: floor(148 / tiles),
// at most 16 and at most the k-block count; every split gets at least one k-block.
inline void gb_split(int64_t M, int64_t N, int64_t K, int& splits, int& kbc) {
  const int64_t tiles = ((M + gb::BM - 1) / gb::BM) * ((N + gb::BN - 1) / gb::BN);
  const int64_t nkb = std::max<int64_t>((K + gb::BK - 1) / gb::BK, 1);
  int64_t sp = std::max<int64_t>(148 / std::max<int64_t>(tiles, 1), 1);
  sp = std::min<int64_t>(sp, std::min<int64_t>(nkb, 16));
  kbc = (int)((nkb + sp - 1) / sp);
  splits = (int)((nkb + kbc - 1) / kbc);
}
inline LinBwdPlan lin_bwd_plan(int64_t m, int32_t k, int32_t n) {
  LinBwdPlan P;
  memset(&P, 0, sizeof(P));
  P.ld_n = ((int64_t)n + 7) / 8 * 8;
  P.ld_m = (m + 7) / 8 * 8;
  P.rho = 0;
  P.mux = align256((size_t)m * 4);
  const size_t base = 2 * align256((size_t)m * 4);
  size_t o = base;
  P.dr_hi = o; o += align256((size_t)m * P.ld_n * 2);
  P.dr_lo = o; o += align256((size_t)m * P.ld_n * 2);
  P.tt = o; o += align256((size_t)k * P.ld_n * 2);
  gb_split(m, k, n, P.dr_split, P.dr_kbc);
  P.dr_part = o;
  if (P.dr_split > 1) o += align256((size_t)P.dr_split * m * k * 4);
  const size_t end_dr = o;
  o = base;
  P.dw_hi = o; o += align256((size_t)n * P.ld_m * 2);
  P.dw_lo = o; o += align256((size_t)n * P.ld_m * 2);
  P.qt = o; o += align256((size_t)k * P.ld_m * 2);
  gb_split(n, k, m, P.dw_split, P.dw_kbc);
  P.dw_part = o;
  if (P.dw_split > 1) o += align256((size_t)P.dw_split * n * k * 4);
  // rho, the gain's gradient and dx: row blocks of at least 16 rows, at most 2048 blocks, each
  // leaving one partial row of the gain's gradient (between the two products, so it reuses the
  // same space)
  P.dnw_split = (int)std::max<int64_t>(std::min<int64_t>((m + 15) / 16, 2048), 1);
  P.dnw_rows = (int)std::max<int64_t>((m + P.dnw_split - 1) / P.dnw_split, 1);
  P.dnw_part = base;
  const size_t end_dnw = base + align256((size_t)P.dnw_split * k * 4);
  P.bytes = std::max(std::max(end_dr, o), end_dnw);
  return P;
}

extern "C" {

int32_t mmf_packed_row_words(int32_t k) { return k <= 0 ? 0 : row_words(k); }

size_t mmf_packed_words(int32_t n, int32_t k) {
  return (n <= 0 || k <= 0) ? 0 : (size_t)n * (size_t)row_words(k);
}


size_t mmf_workspace_bytes(mmf_op op, int64_t m, int32_t d, int32_t inner, int32_t n_layers) {
  if (m < 0 || d < 0 || inner < 0) return 0;
  switch (op) {
    case MMF_OP_PACK:
      return align256(kPackSumBlocks * sizeof(double));
    case MMF_OP_BITLINEAR:
      return d > 0 ? align256((size_t)m * row_q(d)) + align256((size_t)m * sizeof(float)) : 0;
    case MMF_OP_BLOCK:
      return block_ws(nullptr, m, d, inner, MMF_F32).bytes;
    case MMF_OP_SCAN:
      return d > 0 ? scan_ws_bytes(m, d) : 0;
    case MMF_OP_HEAD:
      return inner > 0 ? head_ws_bytes(inner, d) : 0;
    case MMF_OP_BITLINEAR_BWD:
      return d > 0 && inner > 0 ? lin_bwd_plan(m, d, inner).bytes : 0;
    case MMF_OP_DECODE:
      return decode_ws_head(m, d, inner) + 2 * align256((size_t)m * d * 4);
    case MMF_OP_STACK:
      return block_ws(nullptr, m, d, inner, MMF_F32).bytes + 2 * align256((size_t)m * d * 4);
  }
  return 0;
}

mmf_status mmf_pack_ternary(const void* w, mmf_dtype w_dtype, int32_t n, int32_t k,
                            uint32_t* codes_out, float* scale_out, void* ws, size_t ws_bytes,
                            mmf_stream_t stream) {
  MMF_CHECK_ARG(n > 0 && k > 0, "pack: bad shape [%d][%d]", n, k);
  MMF_CHECK_ARG(valid_dtype(w_dtype), "pack: bad dtype %d", (int)w_dtype);
  MMF_CHECK_ARG(w && codes_out && scale_out, "pack: null pointer");
  MMF_CHECK_ARG(aligned16(codes_out), "pack: codes_out not 16-byte aligned");
  MMF_TRY(check_ws(ws, ws_bytes, mmf_workspace_bytes(MMF_OP_PACK, (int64_t)n * k, 0, 0, 0)));
  DevInfo* di;
  MMF_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  double* partial = reinterpret_cast<double*>(ws);
  const int64_t count = (int64_t)n * k;
  const int32_t kw = row_words(k);
  const int64_t words = (int64_t)n * kw;
  const unsigned pgrid = (unsigned)std::min<int64_t>((words + 255) / 256, (int64_t)di->sms * 16);
  LaunchScope ls(MMF_KERNEL_OTHER, (double)count * 2.0 * dsize(w_dtype) + (double)words * 4.0, st);
  g_launches.fetch_add(2);  // three kernels under one timing scope
  if (w_dtype == MMF_F32) {
    pack_abssum_kernel<MMF_F32><<<kPackSumBlocks, 256, 0, st>>>(reinterpret_cast<const float*>(w), count, partial);
    MMF_TRY(check_launch("pack_abssum_kernel"));
    pack_scale_kernel<<<1, 32, 0, st>>>(partial, kPackSumBlocks, count, scale_out);
    MMF_TRY(check_launch("pack_scale_kernel"));
    pack_codes_kernel<MMF_F32><<<pgrid, 256, 0, st>>>(reinterpret_cast<const float*>(w), n, k, kw, scale_out, codes_out);
  } else {
    pack_abssum_kernel<MMF_BF16><<<kPackSumBlocks, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(w), count, partial);
    MMF_TRY(check_launch("pack_abssum_kernel"));
    pack_scale_kernel<<<1, 32, 0, st>>>(partial, kPackSumBlocks, count, scale_out);
    MMF_TRY(check_launch("pack_scale_kernel"));
    pack_codes_kernel<MMF_BF16><<<pgrid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(w), n, k, kw, scale_out, codes_out);
  }
  return check_launch("pack_codes_kernel");
}

mmf_status mmf_bitlinear_fwd(const void* x, mmf_dtype x_dtype, int64_t m, const float* norm_w,
                             const mmf_ternary* w, void* y, mmf_dtype y_dtype, int8_t* q_dbg,
                             float* deq_dbg, int32_t* acc_dbg, void* ws, size_t ws_bytes,
                             mmf_stream_t stream) {
  MMF_CHECK_ARG(m >= 0, "bitlinear: negative m");
  MMF_CHECK_ARG(valid_dtype(x_dtype) && valid_dtype(y_dtype), "bitlinear: bad dtype");
  MMF_CHECK_ARG(w != nullptr && w->n > 0 && w->k > 0 && w->k <= 32768, "bitlinear: bad weight descriptor");
  MMF_TRY(check_ternary(w, w->n, w->k, "bitlinear"));
  if (m == 0) return MMF_OK;
  MMF_CHECK_ARG(x && y, "bitlinear: null x or y");
  MMF_CHECK_ARG(aligned16(x) && aligned16(y), "bitlinear: x / y not 16-byte aligned");
  MMF_TRY(check_ws(ws, ws_bytes, mmf_workspace_bytes(MMF_OP_BITLINEAR, m, w->k, w->n, 0)));
  DevInfo* di;
  MMF_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t ldq = row_q(w->k);
  int8_t* q = reinterpret_cast<int8_t*>(ws);
  float* deq = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + align256((size_t)m * ldq));
  NormQuantArgs nq;
  memset(&nq, 0, sizeof(nq));
  nq.x = x; nq.ldx = w->k; nq.xdt = x_dtype; nq.m = m; nq.k = w->k; nq.eps = 1e-8f; nq.ngain = 1;
  nq.gain[0] = norm_w; nq.q[0] = q; nq.deq[0] = deq; nq.ldq = ldq;
  MMF_TRY(launch_norm_quant(nq, kRowPlain, st));
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.m = m; g.k = w->k; g.kw = row_words(w->k); g.ldq = ldq; g.ydt = y_dtype; g.nseg = 1;
  g.seg[0] = make_seg(q, deq, *w, y, w->n, 0, nullptr, 0, acc_dbg, w->n);
  MMF_TRY(launch_gemm(g, *di, st));
  if (q_dbg) {
    cudaError_t e = cudaMemcpy2DAsync(q_dbg, w->k, q, ldq, w->k, m, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "cudaMemcpy2DAsync: %s", cudaGetErrorString(e));
  }
  if (deq_dbg) {
    cudaError_t e = cudaMemcpyAsync(deq_dbg, deq, m * sizeof(float), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "cudaMemcpyAsync: %s", cudaGetErrorString(e));
  }
  return MMF_OK;
}

mmf_status mmf_bitlinear_fwd_noalloc(const void* x, mmf_dtype x_dtype, int64_t m, const float* norm_w,
                                     const mmf_ternary* w, void* y, mmf_dtype y_dtype,
                                     mmf_stream_t stream) {
  MMF_CHECK_ARG(m >= 0, "bitlinear_noalloc: negative m");
  MMF_CHECK_ARG(w != nullptr && w->n > 0 && w->k > 0, "bitlinear_noalloc: bad weight descriptor");
  if (m == 0) return MMF_OK;
  const size_t need = mmf_workspace_bytes(MMF_OP_BITLINEAR, m, w->k, w->n, 0);
  if (need > (size_t)MMF_NOALLOC_SCRATCH_BYTES)
    return fail(MMF_ERR_WORKSPACE,
                "bitlinear_noalloc: m=%lld rows of K=%d need %zu bytes of scratch; the static array "
                "holds %u bytes (use mmf_bitlinear_fwd with a workspace, or fewer rows per call)",
                (long long)m, w->k, need, (unsigned)MMF_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  MMF_TRY(noalloc_scratch(&scratch));
  return mmf_bitlinear_fwd(x, x_dtype, m, norm_w, w, y, y_dtype, nullptr, nullptr, nullptr, scratch,
                           (size_t)MMF_NOALLOC_SCRATCH_BYTES, stream);
}

mmf_status mmf_hgrn_scan(const void* zf, const void* zi, mmf_dtype z_dtype, int64_t z_stride,
                         int32_t b, int64_t t, int32_t d, const float* h0, void* h_out,
                         mmf_dtype h_dtype, float* h_last, void* ws, size_t ws_bytes,
                         mmf_stream_t stream) {
  MMF_CHECK_ARG(b >= 0 && t >= 0 && d >= 0, "scan: negative size");
  MMF_CHECK_ARG(valid_dtype(z_dtype) && valid_dtype(h_dtype), "scan: bad dtype");
  MMF_CHECK_ARG(z_stride >= d, "scan: z_stride %lld < d %d", (long long)z_stride, d);
  if ((int64_t)b * d == 0) return MMF_OK;
  MMF_CHECK_ARG(t == 0 || (zf && zi && h_out), "scan: null pointer");
  if (t > 16) MMF_TRY(check_ws(ws, ws_bytes, scan_ws_bytes((int64_t)b * t, d)));
  DevInfo* di;
  MMF_TRY(device_info(&di));
  ScanArgs a;
  memset(&a, 0, sizeof(a));
  a.zf = zf; a.zi = zi; a.zdt = z_dtype; a.zstride = z_stride; a.b = b; a.t = t; a.d = d;
  a.h0 = h0; a.h = h_out; a.hdt = h_dtype; a.h_last = h_last;
  return launch_scan(a, ws, reinterpret_cast<cudaStream_t>(stream));
}

mmf_status mmf_block_fwd(const mmf_block_weights* w, const void* x, mmf_dtype dtype, int32_t b,
                         int64_t t, const float* h0, void* y, float* h_last, void* ws,
                         size_t ws_bytes, mmf_stream_t stream) {
  MMF_TRY(check_block(w));
  MMF_CHECK_ARG(valid_dtype(dtype), "block: bad dtype");
  MMF_CHECK_ARG(b >= 0 && t >= 0, "block: negative size");
  const int64_t m = (int64_t)b * t;
  if (m == 0) {
    if (b > 0 && h_last) {
      DevInfo* di;
      MMF_TRY(device_info(&di));
      ScanArgs a;
      memset(&a, 0, sizeof(a));
      a.b = b; a.t = 0; a.d = w->d; a.h0 = h0; a.h_last = h_last;
      return launch_scan(a, nullptr, reinterpret_cast<cudaStream_t>(stream));
    }
    return MMF_OK;
  }
  MMF_CHECK_ARG(x && y && x != y, "block: null or aliased x / y");
  MMF_CHECK_ARG(aligned16(x) && aligned16(y), "block: x / y not 16-byte aligned");
  MMF_TRY(check_ws(ws, ws_bytes, mmf_workspace_bytes(MMF_OP_BLOCK, m, w->d, w->inner, 1)));
  DevInfo* di;
  MMF_TRY(device_info(&di));
  const BlockWs W = block_ws(ws, m, w->d, w->inner, dtype);
  return run_block(w, x, dtype, b, t, h0, y, h_last, W, *di, reinterpret_cast<cudaStream_t>(stream));
}

mmf_status mmf_block_fwd_taps(const mmf_block_weights* w, const void* x, mmf_dtype dtype, int32_t b,
                              int64_t t, const float* h0, void* y, float* h_last,
                              const mmf_block_taps* taps, void* ws, size_t ws_bytes,
                              mmf_stream_t stream) {
  MMF_CHECK_ARG(taps != nullptr, "block taps: null taps");
  MMF_TRY(mmf_block_fwd(w, x, dtype, b, t, h0, y, h_last, ws, ws_bytes, stream));
  const int64_t m = (int64_t)b * t;
  if (m == 0) return MMF_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const BlockWs W = block_ws(ws, m, w->d, w->inner, dtype);
  const int32_t d = w->d, inner = w->inner;
  const size_t es = dsize(dtype);
  auto copy2d = [&](void* dst, size_t dpitch, const void* src, size_t spitch, size_t width, size_t rows) -> mmf_status {
    if (!dst) return MMF_OK;
    cudaError_t e = cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, rows, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "taps copy: %s", cudaGetErrorString(e));
    return MMF_OK;
  };
  MMF_TRY(copy2d(taps->q_ifg, d, W.q3, row_q(d), d, 3 * m));
  MMF_TRY(copy2d(taps->deq_ifg, 3 * m * 4, W.deq, 3 * m * 4, 3 * m * 4, 1));
  for (int p = 0; p < 3; ++p)  // the [i | f | g] planes into the [m][3d] tap
    MMF_TRY(copy2d(taps->z ? reinterpret_cast<uint8_t*>(taps->z) + p * d * es : nullptr, 3 * d * es,
                   reinterpret_cast<const uint8_t*>(W.z) + p * (size_t)m * d * es, d * es, d * es, m));
  MMF_TRY(copy2d(taps->h, d * es, W.h, d * es, d * es, m));
  MMF_TRY(copy2d(taps->q_o, d, W.qo, row_q(d), d, m));
  MMF_TRY(copy2d(taps->deq_o, m * 4, W.deq + 3 * m, m * 4, m * 4, 1));
  MMF_TRY(copy2d(taps->x1, d * es, W.x1, d * es, d * es, m));
  MMF_TRY(copy2d(taps->q_gate, d, W.qg, row_q(d), d, m));
  MMF_TRY(copy2d(taps->deq_gate, m * 4, W.deq + 4 * m, m * 4, m * 4, 1));
  if (glu_fused(m, inner)) MMF_TRY(copy2d(taps->v, inner * es, W.gu, inner * es, inner * es, m));
  else MMF_TRY(copy2d(taps->gu, 2 * inner * es, W.gu, 2 * inner * es, 2 * inner * es, m));
  MMF_TRY(copy2d(taps->q_down, inner, W.qd, row_q(inner), inner, m));
  MMF_TRY(copy2d(taps->deq_down, m * 4, W.deq + 5 * m, m * 4, m * 4, 1));
  return MMF_OK;
}

}  // extern "C"

namespace {

// ---------------------------------------------------------------------------------------------
// fused decode (up to 8 token rows on the CUDA-core engine): four launches per block
// ---------------------------------------------------------------------------------------------
// Measured on the 2.7B shape (32 blocks): 1.24 / 1.75 / 2.64 ms per step at 2 / 4 / 8 rows against
// 2.20 ms for the block path on the tensor-core GEMMs, so the automatic engine choice (8 rows and
// up on the tensor cores) leaves 1, 2 and 4 rows here; 8 rows come here only on the CUDA-core
// engine.
bool decode_fused(int32_t b, int32_t d, int32_t inner) {
  // 1, 2, 4 or 8 token rows (the kernel's compile-time row count must equal b)
  if ((b != 1 && b != 2 && b != 4 && b != 8) || use_tensor_path(b)) return false;
  if (d % 8 || inner % 8) return false;
  return true;
}

// Channels per CTA: about one CTA per SM, fewer channels when the weight slice would not fit.
int dec_chan_per_cta(int mode, int nout, int nmat, int kw, int k, int ngain, int b, int sms) {
  int cpc = std::max(1, (nout + sms - 1) / sms);
  while (cpc > 1 && dec::smem_layout(mode, nmat, cpc, kw, k, ngain, b).total > (size_t)dec::kMaxSmem) cpc = (cpc + 1) / 2;
  return cpc;
}

mmf_status launch_dec(dec::Args& a, const DevInfo& di, cudaStream_t st) {
  a.chan_per_cta = dec_chan_per_cta(a.mode, a.nout, a.nmat, a.kw, a.k, a.ngain, a.b, di.sms);
  const dec::Smem L = dec::smem_layout(a.mode, a.nmat, a.chan_per_cta, a.kw, a.k, a.ngain, a.b);
  if (L.total > (size_t)dec::kMaxSmem) return fail(MMF_ERR_UNSUPPORTED, "decode: K=%d too large for one CTA", a.k);
  a.wait_limit_us = g_wait_limit.load();
  const dim3 grid((unsigned)((a.nout + a.chan_per_cta - 1) / a.chan_per_cta));
  double bytes = 0;
  for (int j = 0; j < a.nmat; ++j) bytes += (double)a.nout * a.kw * 4.0;
  LaunchScope ls(MMF_KERNEL_GEMM_SIMT, bytes, st);
  if (a.b != 1 && a.b != 2 && a.b != 4 && a.b != 8)
    return fail(MMF_ERR_UNSUPPORTED, "fused decode takes 1, 2, 4 or 8 token rows, got %d", a.b);
  // token rows as a compile-time count: 1, 2, 4 or 8 (decode_fused admits no other count)
#define MMF_DEC(XT_, NB_) launch_k(dec::dec_proj_kernel<XT_, NB_>, grid, dim3(dec::kThreads), L.total, st, a)
  if (a.xdt == MMF_F32) {
    if (a.b == 1) MMF_DEC(MMF_F32, 1);
    else if (a.b == 2) MMF_DEC(MMF_F32, 2);
    else if (a.b == 4) MMF_DEC(MMF_F32, 4);
    else MMF_DEC(MMF_F32, 8);
  } else {
    if (a.b == 1) MMF_DEC(MMF_BF16, 1);
    else if (a.b == 2) MMF_DEC(MMF_BF16, 2);
    else if (a.b == 4) MMF_DEC(MMF_BF16, 4);
    else MMF_DEC(MMF_BF16, 8);
  }
#undef MMF_DEC
  return check_launch("dec_proj_kernel");
}

mmf_status tap_copy(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  if (!dst || bytes == 0) return MMF_OK;
  cudaError_t e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "taps copy: %s", cudaGetErrorString(e));
  return MMF_OK;
}
mmf_status tap_copy2d(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width, size_t rows,
                      cudaStream_t st) {
  if (!dst || width == 0 || rows == 0) return MMF_OK;
  cudaError_t e = cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, rows, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "taps copy: %s", cudaGetErrorString(e));
  return MMF_OK;
}
// dst[r][c] = float(src[r][c]) (debug taps).
mmf_status tap_to_f32(float* dst, int64_t dst_ld, const void* src, mmf_dtype sdt, int64_t src_ld, int64_t rows,
                      int32_t cols, cudaStream_t st) {
  if (!dst || rows * cols == 0) return MMF_OK;
  const int64_t blocks = std::min<int64_t>((rows * cols + 255) / 256, 4096);
  launch_k(tap_to_f32_kernel, dim3((unsigned)blocks), dim3(256), 0, st, src, sdt, rows, cols, src_ld, dst, dst_ld);
  return check_launch("tap_to_f32_kernel");
}

// One block, one token per row: x [b][d] -> y [b][d], state [b][d] updated in place. Scratch:
// h and g (float32, [b][d]), x1 [b][d] and v [b][inner] (dtype). `tp` (nullable) receives the
// step's intermediates.
mmf_status run_block_decode(const mmf_block_weights* w, const void* x, mmf_dtype dt, int32_t b, float* state,
                            void* y, uint8_t* scratch, const DevInfo& di, cudaStream_t st,
                            const mmf_decode_taps* tp = nullptr) {
  const int32_t d = w->d, inner = w->inner;
  float* h32 = reinterpret_cast<float*>(scratch);
  float* g32 = reinterpret_cast<float*>(scratch + align256((size_t)b * d * 4));
  void* x1 = scratch + 2 * align256((size_t)b * d * 4);
  void* v = scratch + 3 * align256((size_t)b * d * 4);
  dec::Args a;
  memset(&a, 0, sizeof(a));
  a.b = b; a.eps = w->eps; a.xdt = dt; a.ydt = dt;
  // i/f/g + gates + recurrence step
  a.mode = dec::kIFG; a.k = d; a.kw = row_words(d); a.nout = d; a.nmat = 3; a.ngain = 3;
  a.w[0] = w->i.codes; a.w[1] = w->f.codes; a.w[2] = w->g.codes;
  a.sw[0] = w->i.scale; a.sw[1] = w->f.scale; a.sw[2] = w->g.scale;
  a.gain[0] = w->nw_i; a.gain[1] = w->nw_f; a.gain[2] = w->nw_g;
  a.x = x; a.y = h32; a.g_out = g32; a.state = state;
  if (tp) { a.q_tap = tp->q_ifg; a.deq_tap = tp->deq_ifg; a.z_tap = tp->z; }
  MMF_TRY(launch_dec(a, di, st));
  if (tp) MMF_TRY(tap_copy(tp->h, h32, (size_t)b * d * 4, st));
  // g_norm + o_proj + residual
  memset(&a, 0, sizeof(a));
  a.b = b; a.eps = w->eps; a.xdt = dt; a.ydt = dt;
  a.mode = dec::kO; a.k = d; a.kw = row_words(d); a.nout = d; a.nmat = 1; a.ngain = 1;
  a.w[0] = w->o.codes; a.sw[0] = w->o.scale; a.gain[0] = w->nw_o;
  a.h = h32; a.gin = g32; a.gnorm_w = w->gnorm_w; a.res = x; a.y = x1;
  if (tp) { a.q_tap = tp->q_o; a.deq_tap = tp->deq_o; }
  MMF_TRY(launch_dec(a, di, st));
  if (tp) MMF_TRY(tap_copy(tp->x1, x1, (size_t)b * d * dsize(dt), st));
  // gate_proj: v = SiLU(gate) * up
  memset(&a, 0, sizeof(a));
  a.b = b; a.eps = w->eps; a.xdt = dt; a.ydt = dt;
  a.mode = dec::kGate; a.k = d; a.kw = row_words(d); a.nout = inner; a.nmat = 2; a.ngain = 1;
  a.w[0] = w->gate.codes; a.w[1] = w->gate.codes; a.row_off[1] = inner;
  a.sw[0] = w->gate.scale; a.sw[1] = w->gate.scale; a.gain[0] = w->nw_gate;
  a.x = x1; a.y = v;
  if (tp) { a.q_tap = tp->q_gate; a.deq_tap = tp->deq_gate; }
  MMF_TRY(launch_dec(a, di, st));
  if (tp) MMF_TRY(tap_copy(tp->v, v, (size_t)b * inner * dsize(dt), st));
  // down_proj + residual
  memset(&a, 0, sizeof(a));
  a.b = b; a.eps = w->eps; a.xdt = dt; a.ydt = dt;
  a.mode = dec::kDown; a.k = inner; a.kw = row_words(inner); a.nout = d; a.nmat = 1; a.ngain = 1;
  a.w[0] = w->down.codes; a.sw[0] = w->down.scale; a.gain[0] = w->nw_down;
  a.x = v; a.res = x1; a.y = y;
  if (tp) { a.q_tap = tp->q_down; a.deq_tap = tp->deq_down; }
  MMF_TRY(launch_dec(a, di, st));
  if (tp) MMF_TRY(tap_copy(tp->y, y, (size_t)b * d * dsize(dt), st));
  return MMF_OK;
}

// The intermediates of one block path step (run_block with t = 1) into decode taps.
mmf_status block_decode_taps(const mmf_block_weights* w, int32_t b, mmf_dtype dt, const BlockWs& W, const void* y,
                             const mmf_decode_taps* tp, cudaStream_t st) {
  const int64_t m = b;
  const int32_t d = w->d, inner = w->inner;
  const size_t es = dsize(dt);
  MMF_TRY(tap_copy2d(tp->q_ifg, d, W.q3, row_q(d), d, 3 * m, st));
  MMF_TRY(tap_copy(tp->deq_ifg, W.deq, 3 * m * 4, st));
  for (int p = 0; p < 3; ++p)
    MMF_TRY(tap_to_f32(tp->z ? tp->z + p * d : nullptr, 3 * (int64_t)d,
                       reinterpret_cast<const uint8_t*>(W.z) + p * (size_t)m * d * es, dt, d, m, d, st));
  MMF_TRY(tap_to_f32(tp->h, d, W.h, dt, d, m, d, st));
  MMF_TRY(tap_copy2d(tp->q_o, d, W.qo, row_q(d), d, m, st));
  MMF_TRY(tap_copy(tp->deq_o, W.deq + 3 * m, m * 4, st));
  MMF_TRY(tap_copy(tp->x1, W.x1, m * d * es, st));
  MMF_TRY(tap_copy2d(tp->q_gate, d, W.qg, row_q(d), d, m, st));
  MMF_TRY(tap_copy(tp->deq_gate, W.deq + 4 * m, m * 4, st));
  if (glu_fused(m, inner)) MMF_TRY(tap_copy(tp->v, W.gu, m * inner * es, st));
  else MMF_TRY(tap_copy(tp->gu, W.gu, m * 2 * inner * es, st));
  MMF_TRY(tap_copy2d(tp->q_down, inner, W.qd, row_q(inner), inner, m, st));
  MMF_TRY(tap_copy(tp->deq_down, W.deq + 5 * m, m * 4, st));
  return tap_copy(tp->y, y, m * d * es, st);
}

// The quantisation of a decode step's input with layer w's three i / f / g gains (row stage).
mmf_status sk_quant_in(const mmf_block_weights* w, const void* x, mmf_dtype dt, int32_t b, const SkWs& S,
                       cudaStream_t st) {
  drow::Args a;
  memset(&a, 0, sizeof(a));
  a.mode = drow::kQuantIn; a.d = w->d; a.inner = w->inner; a.eps = w->eps; a.dt = dt; a.x = x;
  a.ngain = 3; a.ldq = row_q(w->d);
  a.gain[0] = w->nw_i; a.gain[1] = w->nw_f; a.gain[2] = w->nw_g;
  for (int j = 0; j < 3; ++j) { a.q[j] = S.q3 + (int64_t)j * b * a.ldq; a.deq[j] = S.deq + j * b; }
  return launch_row_stage(a, b, st);
}

// One block of a decode step on the skinny tensor-core path: four products (each one launch of
// the skinny kernel into exact int32 accumulators) and four row stages (the products' epilogues:
// gates and the recurrence step, residuals, GLU; each quantising the next product's input). The
// codes of x for this layer are in S.q3 / S.deq[0..3b) on entry; on exit they hold the codes of y
// for `next` (the following layer, or none). `tp` (nullable) receives the intermediates.
mmf_status run_block_decode_sk(const mmf_block_weights* w, const mmf_block_weights* next, const void* x,
                               mmf_dtype dt, int32_t b, float* state, void* y, const SkWs& S, const DevInfo& di,
                               cudaStream_t st, const mmf_decode_taps* tp) {
  const int32_t d = w->d, inner = w->inner;
  const int64_t ldq_d = row_q(d), ldq_i = row_q(inner);
  const size_t es = dsize(dt);
  if (tp) {
    MMF_TRY(tap_copy2d(tp->q_ifg, d, S.q3, ldq_d, d, 3 * (size_t)b, st));
    MMF_TRY(tap_copy(tp->deq_ifg, S.deq, 3 * (size_t)b * 4, st));
  }
  // i / f / g products: acc = [zi | zf | g] accumulators
  SkSeg g3[3] = {{S.q3, w->i.codes, d, S.acc},
                 {S.q3 + (int64_t)b * ldq_d, w->f.codes, d, S.acc + d},
                 {S.q3 + 2 * (int64_t)b * ldq_d, w->g.codes, d, S.acc + 2 * d}};
  MMF_TRY(launch_skinny(g3, 3, b, d, ldq_d, 3 * (int64_t)d, di, st));
  drow::Args a;
  memset(&a, 0, sizeof(a));
  a.mode = drow::kIFG; a.d = d; a.inner = inner; a.eps = w->eps; a.dt = dt; a.acc = S.acc; a.ldacc = 3 * (int64_t)d;
  a.deq_in[0] = S.deq; a.deq_in[1] = S.deq + b; a.deq_in[2] = S.deq + 2 * b;
  a.sw[0] = w->i.scale; a.sw[1] = w->f.scale; a.sw[2] = w->g.scale;
  a.state = state; a.gnorm_w = w->gnorm_w;
  a.ngain = 1; a.gain[0] = w->nw_o; a.q[0] = S.qo; a.ldq = ldq_d; a.deq[0] = S.deq + 3 * b;
  if (tp) { a.z_tap = tp->z; a.h_tap = tp->h; }
  MMF_TRY(launch_row_stage(a, b, st));
  if (tp) {
    MMF_TRY(tap_copy2d(tp->q_o, d, S.qo, ldq_d, d, b, st));
    MMF_TRY(tap_copy(tp->deq_o, S.deq + 3 * b, (size_t)b * 4, st));
  }
  // o_proj, then x1 = x + o and gate_proj's codes
  SkSeg go = {S.qo, w->o.codes, d, S.acc};
  MMF_TRY(launch_skinny(&go, 1, b, d, ldq_d, d, di, st));
  memset(&a, 0, sizeof(a));
  a.mode = drow::kO; a.d = d; a.inner = inner; a.eps = w->eps; a.dt = dt; a.acc = S.acc; a.ldacc = d;
  a.deq_in[0] = S.deq + 3 * b; a.sw[0] = w->o.scale; a.res = x; a.out = S.x1;
  a.ngain = 1; a.gain[0] = w->nw_gate; a.q[0] = S.qg; a.ldq = ldq_d; a.deq[0] = S.deq + 4 * b;
  MMF_TRY(launch_row_stage(a, b, st));
  if (tp) {
    MMF_TRY(tap_copy(tp->x1, S.x1, (size_t)b * d * es, st));
    MMF_TRY(tap_copy2d(tp->q_gate, d, S.qg, ldq_d, d, b, st));
    MMF_TRY(tap_copy(tp->deq_gate, S.deq + 4 * b, (size_t)b * 4, st));
  }
  // gate_proj ([gate | up] accumulators), then v = SiLU(gate) * up and down_proj's codes
  SkSeg gg = {S.qg, w->gate.codes, 2 * inner, S.acc};
  MMF_TRY(launch_skinny(&gg, 1, b, d, ldq_d, 2 * (int64_t)inner, di, st));
  memset(&a, 0, sizeof(a));
  a.mode = drow::kGate; a.d = d; a.inner = inner; a.eps = w->eps; a.dt = dt; a.acc = S.acc; a.ldacc = 2 * (int64_t)inner;
  a.deq_in[0] = S.deq + 4 * b; a.sw[0] = w->gate.scale; a.out = S.v;
  a.ngain = 1; a.gain[0] = w->nw_down; a.q[0] = S.qd; a.ldq = ldq_i; a.deq[0] = S.deq + 5 * b;
  MMF_TRY(launch_row_stage(a, b, st));
  if (tp) {
    MMF_TRY(tap_copy(tp->v, S.v, (size_t)b * inner * es, st));
    MMF_TRY(tap_copy2d(tp->q_down, inner, S.qd, ldq_i, inner, b, st));
    MMF_TRY(tap_copy(tp->deq_down, S.deq + 5 * b, (size_t)b * 4, st));
  }
  // down_proj, then y = x1 + down and the next layer's input codes
  SkSeg gd = {S.qd, w->down.codes, d, S.acc};
  MMF_TRY(launch_skinny(&gd, 1, b, inner, ldq_i, d, di, st));
  memset(&a, 0, sizeof(a));
  a.mode = drow::kDown; a.d = d; a.inner = inner; a.eps = w->eps; a.dt = dt; a.acc = S.acc; a.ldacc = d;
  a.deq_in[0] = S.deq + 5 * b; a.sw[0] = w->down.scale; a.res = S.x1; a.out = y;
  if (next) {
    a.ngain = 3; a.ldq = ldq_d;
    a.gain[0] = next->nw_i; a.gain[1] = next->nw_f; a.gain[2] = next->nw_g;
    for (int j = 0; j < 3; ++j) { a.q[j] = S.q3 + (int64_t)j * b * ldq_d; a.deq[j] = S.deq + j * b; }
  }
  MMF_TRY(launch_row_stage(a, b, st));
  if (tp) MMF_TRY(tap_copy(tp->y, y, (size_t)b * d * es, st));
  return MMF_OK;
}

// Which decode path a step of b rows takes (the automatic choice and the forced ones).
enum DecodePath { kDecFused = 0, kDecSkinny = 1, kDecBlock = 2 };
int decode_path_for(int32_t b, int32_t d, int32_t inner) {
  const int p = g_decode_path.load();
  const bool sk_ok = b >= 1 && b <= 64 && d <= drow::kMaxK && inner <= drow::kMaxK && d % 8 == 0 && inner % 8 == 0;
  if (p == MMF_DECODE_SKINNY) return sk_ok ? kDecSkinny : kDecBlock;
  if (p == MMF_DECODE_BLOCK) return kDecBlock;
  if (p == MMF_DECODE_FUSED) return (b == 1 || b == 2 || b == 4 || b == 8) && d % 8 == 0 && inner % 8 == 0 ? kDecFused
                                                                                                              : kDecBlock;
  // automatic: the engine setting first (the CUDA-core engine keeps the fused path, the
  // tensor-core engine the block path), then the row count. Measured on the 2.7B shape (8 layers,
  // graph replay): fused 0.244 ms at 1 row against 0.377 ms skinny; skinny 0.373 / 0.468 ms at
  // 8 / 64 rows against 0.52 / 0.53 ms on the block path.
  if (g_gemm_path.load() == MMF_GEMM_SIMT) return decode_fused(b, d, inner) ? kDecFused : kDecBlock;
  if (g_gemm_path.load() == MMF_GEMM_TENSOR) return kDecBlock;
  if ((b == 1 || b == 2) && d % 8 == 0 && inner % 8 == 0) return kDecFused;
  return sk_ok ? kDecSkinny : kDecBlock;
}

// The fused decode paths bulk-copy the norm gains: every gain vector must start on 16 bytes.
bool gains_aligned(const mmf_block_weights* layers, int32_t n_layers) {
  for (int l = 0; l < n_layers; ++l) {
    const float* g[7] = {layers[l].nw_i, layers[l].nw_f, layers[l].nw_g, layers[l].nw_o,
                         layers[l].nw_gate, layers[l].nw_down, layers[l].gnorm_w};
    for (const float* p : g)
      if (p && (reinterpret_cast<uintptr_t>(p) & 15u)) return false;
  }
  return true;
}

mmf_status decode_impl(const mmf_block_weights* layers, int32_t n_layers, const void* x, mmf_dtype dtype, int32_t b,
                       float* state, void* y, const mmf_decode_taps* taps, void* ws, size_t ws_bytes,
                       mmf_stream_t stream) {
  MMF_CHECK_ARG(layers != nullptr && n_layers > 0, "decode: no layers");
  MMF_CHECK_ARG(valid_dtype(dtype), "decode: bad dtype");
  MMF_CHECK_ARG(b >= 0, "decode: negative batch");
  for (int l = 0; l < n_layers; ++l) {
    MMF_TRY(check_block(&layers[l]));
    MMF_CHECK_ARG(layers[l].d == layers[0].d && layers[l].inner == layers[0].inner,
                  "decode: layer %d has a different shape", l);
  }
  if (b == 0) return MMF_OK;
  MMF_CHECK_ARG(x && y && state && x != y, "decode: null or aliased pointer");
  MMF_CHECK_ARG(aligned16(x) && aligned16(y), "decode: x / y not 16-byte aligned");
  const int32_t d = layers[0].d, inner = layers[0].inner;
  MMF_TRY(check_ws(ws, ws_bytes, mmf_workspace_bytes(MMF_OP_DECODE, b, d, inner, n_layers)));
  DevInfo* di;
  MMF_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const BlockWs W = block_ws(ws, b, d, inner, dtype);
  const SkWs S = sk_ws(ws, b, d, inner);
  uint8_t* pp = reinterpret_cast<uint8_t*>(ws) + decode_ws_head(b, d, inner);
  void* buf[2] = {pp, pp + align256((size_t)b * d * 4)};
  const void* cur = x;
  int path = decode_path_for(b, d, inner);
  // the fused path bulk-copies the input rows and the gains; the row stages read gains as float4
  if ((path == kDecFused || path == kDecSkinny) && !(al16(x) && gains_aligned(layers, n_layers))) path = kDecBlock;
  if (path == kDecSkinny) MMF_TRY(sk_quant_in(&layers[0], x, dtype, b, S, st));
  for (int l = 0; l < n_layers; ++l) {
    void* out = (l == n_layers - 1) ? y : buf[l & 1];
    float* st_l = state + (int64_t)l * b * d;
    const mmf_decode_taps* tp = taps ? &taps[l] : nullptr;
    if (path == kDecSkinny) {
      MMF_TRY(run_block_decode_sk(&layers[l], l + 1 < n_layers ? &layers[l + 1] : nullptr, cur, dtype, b, st_l, out,
                                  S, *di, st, tp));
    } else if (path == kDecFused) {
      MMF_TRY(run_block_decode(&layers[l], cur, dtype, b, st_l, out, reinterpret_cast<uint8_t*>(ws), *di, st, tp));
    } else {
      MMF_TRY(run_block(&layers[l], cur, dtype, b, 1, st_l, out, st_l, W, *di, st));
      if (tp) MMF_TRY(block_decode_taps(&layers[l], b, dtype, W, out, tp, st));
    }
    cur = out;
  }
  return MMF_OK;
}

}  // namespace

// D [M][N] (row pitch ldd) = alpha * (Ahi + Alo) . B^T on the bf16 tensor cores; A [M][K] and
// B [N][K] bf16 with row pitches lda, ldb (multiples of 8). Returns the number of launches.
mmf_status launch_bf16_gemm(const void* a_hi, const void* a_lo, int64_t lda, const void* b, int64_t ldb,
                            int64_t M, int64_t N, int64_t K, const float* alpha, float* d, int64_t ldd, int splits,
                            int kbc, float* part, cudaStream_t st, int* launches) {
  gb::Params P;
  memset(&P, 0, sizeof(P));
  MMF_TRY(encode_2d(&P.a_hi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a_hi, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2,
                    gb::BK, gb::BM, CU_TENSOR_MAP_SWIZZLE_128B));
  if (a_lo)
    MMF_TRY(encode_2d(&P.a_lo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a_lo, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2,
                      gb::BK, gb::BM, CU_TENSOR_MAP_SWIZZLE_128B));
  MMF_TRY(encode_2d(&P.b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, b, (uint64_t)K, (uint64_t)N, (uint64_t)ldb * 2, gb::BK,
                    gb::BN, CU_TENSOR_MAP_SWIZZLE_128B));
  P.m = (int32_t)M;
  P.n = (int32_t)N;
  P.num_kb = (int32_t)std::max<int64_t>((K + gb::BK - 1) / gb::BK, 1);
  P.kb_per_cta = kbc;
  P.has_lo = a_lo ? 1 : 0;
  P.alpha = alpha;
  P.d = d;
  P.ldd = ldd;
  P.part = splits > 1 ? part : nullptr;
  P.wait_limit_us = g_wait_limit.load();
  const dim3 grid((unsigned)((N + gb::BN - 1) / gb::BN), (unsigned)((M + gb::BM - 1) / gb::BM), (unsigned)splits);
  launch_k(gb::bf16_gemm_kernel, grid, dim3(gb::THREADS), gb::SMEM_BYTES, st, P);
  ++*launches;
  if (splits > 1) {
    launch_k(gb::bf16_gemm_reduce_kernel, dim3((unsigned)M, (unsigned)((N + 255) / 256)), dim3(256), 0, st, part,
             splits, (int32_t)M, (int32_t)N, alpha, d, ldd);
    ++*launches;
  }
  return MMF_OK;
}

// Steps per chunk of the chunked scan backward: the whole sequence up to 32 steps, 32 up to 4096
// steps, then a multiple of 16 giving at most 128 chunks; so b * nchunk <= ceil(b t / 8) and the
// forward scan's scratch size bounds the three [b][nchunk][d] arrays.
inline int32_t scan_bwd_chunk(int64_t t) {
  if (t <= 32) return (int32_t)t;
  if (t <= 4096) return 32;
  const int64_t c = (t + 127) / 128;
  return (int32_t)((c + 15) / 16 * 16);
}

template <mmf_dtype DT, int VEC>
void scan_bwd_launch(const bwd::ScanBwdArgs& a, cudaStream_t st) {
  const unsigned blocks = (unsigned)((int64_t)a.gx * a.nchunk * a.b);
  if (a.nchunk == 1) {
    launch_k(bwd::scan_bwd_replay_kernel<DT, VEC, true>, dim3(blocks), dim3(bwd::kScanBwdThreads), 0, st, a);
    return;
  }
  launch_k(bwd::scan_bwd_fold_kernel<DT, VEC>, dim3(blocks), dim3(bwd::kScanBwdThreads), 0, st, a);
  const unsigned cb = (unsigned)(((int64_t)a.b * a.d + bwd::kScanBwdThreads - 1) / bwd::kScanBwdThreads);
  launch_k(bwd::scan_bwd_carry_kernel, dim3(cb), dim3(bwd::kScanBwdThreads), 0, st, a);
  launch_k(bwd::scan_bwd_replay_kernel<DT, VEC, false>, dim3(blocks), dim3(bwd::kScanBwdThreads), 0, st, a);
}

extern "C" {

mmf_status mmf_decode_step(const mmf_block_weights* layers, int32_t n_layers, const void* x,
                           mmf_dtype dtype, int32_t b, float* state, void* y, void* ws,
                           size_t ws_bytes, mmf_stream_t stream) {
  return decode_impl(layers, n_layers, x, dtype, b, state, y, nullptr, ws, ws_bytes, stream);
}

mmf_status mmf_decode_step_taps(const mmf_block_weights* layers, int32_t n_layers, const void* x,
                                mmf_dtype dtype, int32_t b, float* state, void* y, const mmf_decode_taps* taps,
                                void* ws, size_t ws_bytes, mmf_stream_t stream) {
  MMF_CHECK_ARG(taps != nullptr, "decode taps: null taps");
  return decode_impl(layers, n_layers, x, dtype, b, state, y, taps, ws, ws_bytes, stream);
}

mmf_status mmf_embed_gather(const int32_t* ids, int64_t m, const void* table, mmf_dtype dtype,
                            int32_t vocab, int32_t d, void* out, mmf_stream_t stream) {
  MMF_CHECK_ARG(m >= 0 && vocab > 0 && d > 0, "embed: bad sizes");
  MMF_CHECK_ARG(valid_dtype(dtype), "embed: bad dtype");
  if (m == 0) return MMF_OK;
  MMF_CHECK_ARG(ids && table && out, "embed: null pointer");
  MMF_CHECK_ARG(aligned16(table) && aligned16(out), "embed: table / out not 16-byte aligned");
  DevInfo* di;
  MMF_TRY(device_info(&di));
  {
    LaunchScope ls(MMF_KERNEL_OTHER, (double)m * d * 2.0 * dsize(dtype) + m * 4.0, reinterpret_cast<cudaStream_t>(stream));
    launch_k(embed_gather_kernel, dim3((unsigned)m), dim3(128), 0, reinterpret_cast<cudaStream_t>(stream), ids, m, table, dtype, vocab, d, out);
  }
  return check_launch("embed_gather_kernel");
}

// ---------------------------------------------------------------------------------------------
// language-model head + greedy next token
// ---------------------------------------------------------------------------------------------
mmf_status mmf_lm_head_argmax(const void* x, mmf_dtype x_dtype, int32_t b, int32_t d, const float* norm_w,
                              float eps, const void* table, mmf_dtype table_dtype, int32_t vocab,
                              int32_t* ids, float* logits, void* ws, size_t ws_bytes, mmf_stream_t stream) {
  MMF_CHECK_ARG(b >= 0 && d > 0 && vocab > 0, "head: bad sizes");
  MMF_CHECK_ARG(d % 8 == 0, "head: d = %d is not a multiple of 8", d);
  MMF_CHECK_ARG(valid_dtype(x_dtype) && valid_dtype(table_dtype), "head: bad dtype");
  MMF_CHECK_ARG((size_t)d * 4 <= 200 * 1024, "head: d = %d too large", d);
  if (b == 0) return MMF_OK;
  MMF_CHECK_ARG(x && table && ids, "head: null pointer");
  MMF_CHECK_ARG(aligned16(x) && aligned16(table) && (!norm_w || aligned16(norm_w)),
                "head: x / table / norm_w not 16-byte aligned");
  MMF_TRY(check_ws(ws, ws_bytes, head_ws_bytes(vocab, d)));
  DevInfo* di;
  MMF_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t parr = head_parts_bytes(vocab);
  float* pmax = reinterpret_cast<float*>(ws);
  int32_t* pidx = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(ws) + parr);
  const size_t xes = dsize(x_dtype);
  if (table_dtype == MMF_BF16 && b >= head::kTcMinRows) {
    // tensor cores: the table streams once per kTcRowsMax token rows
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(ws) + 2 * parr);
    const int passes = (b + head::kTcRowsMax - 1) / head::kTcRowsMax;
    LaunchScope ls(MMF_KERNEL_OTHER, (double)vocab * d * 2.0 * passes + (double)b * vocab * (logits ? 4.0 : 0.0), st);
    for (int r0 = 0; r0 < b; r0 += head::kTcRowsMax) {
      const int nb = std::min(b - r0, head::kTcRowsMax);
      MMF_TRY(head_tc_pass(reinterpret_cast<const uint8_t*>(x) + (size_t)r0 * d * xes, x_dtype, nb, d, norm_w, eps,
                           table, vocab, logits ? logits + (int64_t)r0 * vocab : nullptr, pmax, pidx, xs, ids + r0, st));
      g_launches.fetch_add(3);
    }
    g_launches.fetch_sub(1);  // the timing scope counted one launch itself
    return check_launch("head tensor-core kernels");
  }
  // vocabulary split: a few CTAs per SM, at least kMinRowsPerCta rows each
  int nparts = std::min((vocab + head::kMinRowsPerCta - 1) / head::kMinRowsPerCta, di->sms * 4);
  const int rows_per_cta = (vocab + nparts - 1) / nparts;
  nparts = (vocab + rows_per_cta - 1) / rows_per_cta;
  head::Args a;
  memset(&a, 0, sizeof(a));
  a.xdt = x_dtype; a.d = d; a.norm_w = norm_w; a.eps = eps; a.table = table; a.tdt = table_dtype;
  a.vocab = vocab; a.rows_per_cta = rows_per_cta; a.ld_logits = vocab;
  a.pmax = pmax;
  a.pidx = pidx;
  LaunchScope ls(MMF_KERNEL_OTHER, (double)vocab * d * dsize(table_dtype) * ((b + head::kRows - 1) / head::kRows) +
                 (double)b * vocab * (logits ? 4.0 : 0.0), st);
  // passes of 8, 4, 2, 1 rows (each kernel handles exactly its row count)
  for (int r0 = 0; r0 < b;) {
    const int left = b - r0;
    const int nb = left >= 8 ? 8 : left >= 4 ? 4 : left >= 2 ? 2 : 1;
    a.x = reinterpret_cast<const uint8_t*>(x) + (size_t)r0 * d * xes;
    a.b = nb;
    a.logits = logits ? logits + (int64_t)r0 * vocab : nullptr;
    if (x_dtype == MMF_F32 && table_dtype == MMF_F32) head_launch<MMF_F32, MMF_F32>(a, nb, nparts, ids + r0, st);
    else if (x_dtype == MMF_F32) head_launch<MMF_F32, MMF_BF16>(a, nb, nparts, ids + r0, st);
    else if (table_dtype == MMF_F32) head_launch<MMF_BF16, MMF_F32>(a, nb, nparts, ids + r0, st);
    else head_launch<MMF_BF16, MMF_BF16>(a, nb, nparts, ids + r0, st);
    r0 += nb;
    g_launches.fetch_add(2);
  }
  g_launches.fetch_sub(1);  // the timing scope counted one launch itself
  return check_launch("head kernels");
}

// ---------------------------------------------------------------------------------------------
// packed-code integrity
// ---------------------------------------------------------------------------------------------
mmf_status mmf_validate_packed(const mmf_ternary* w, unsigned long long* bad, mmf_stream_t stream) {
  MMF_CHECK_ARG(w != nullptr && w->codes != nullptr && bad != nullptr, "validate: null pointer");
  MMF_CHECK_ARG(w->n >= 0 && w->k >= 0, "validate: negative shape");
  MMF_CHECK_ARG(aligned16(w->codes), "validate: codes not 16-byte aligned");
  MMF_CHECK_ARG((reinterpret_cast<uintptr_t>(bad) & 7u) == 0, "validate: bad counter not 8-byte aligned");
  DevInfo* di;
  MMF_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  MMF_CUDA(cudaMemsetAsync(bad, 0, sizeof(unsigned long long), st));
  const int32_t kw = w->k > 0 ? row_words(w->k) : 0;
  const int64_t total = (int64_t)w->n * kw;
  if (total == 0) return MMF_OK;
  const int64_t blocks = std::min<int64_t>((total + validate::kThreads - 1) / validate::kThreads, (int64_t)di->sms * 8);
  LaunchScope ls(MMF_KERNEL_OTHER, (double)total * 4.0, st);
  launch_k(validate::validate_packed_kernel, dim3((unsigned)blocks), dim3(validate::kThreads), 0, st, w->codes,
           w->n, w->k, kw, bad);
  return check_launch("validate_packed_kernel");
}

// ---------------------------------------------------------------------------------------------
// gradients of the HGRN scan with its gates
// ---------------------------------------------------------------------------------------------
mmf_status mmf_hgrn_scan_backward(const void* zf, const void* zi, const void* h, const void* dh, mmf_dtype dtype,
                                  int32_t b, int64_t t, int32_t d, const float* h0, void* dzf, void* dzi,
                                  float* dh0, void* ws, size_t ws_bytes, mmf_stream_t stream) {
  MMF_CHECK_ARG(b >= 0 && t >= 0 && d >= 0, "scan backward: negative size");
  MMF_CHECK_ARG(valid_dtype(dtype), "scan backward: bad dtype");
  if ((int64_t)b * d == 0) return MMF_OK;
  MMF_CHECK_ARG(t == 0 || (zf && zi && h && dh && dzf && dzi), "scan backward: null pointer");
  const int32_t chunk = t > 0 ? scan_bwd_chunk(t) : 1;
  const int32_t nchunk = (int32_t)((t + chunk - 1) / chunk);
  if (nchunk > 1) MMF_TRY(check_ws(ws, ws_bytes, scan_ws_bytes((int64_t)b * t, d)));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DevInfo* di;
  MMF_TRY(device_info(&di));
  if (t == 0) {
    // no steps: nothing reaches h0
    if (dh0) {
      cudaError_t e = cudaMemsetAsync(dh0, 0, (size_t)b * d * sizeof(float), st);
      if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    }
    return MMF_OK;
  }
  bwd::ScanBwdArgs a;
  memset(&a, 0, sizeof(a));
  a.zf = zf; a.zi = zi; a.h = h; a.dh = dh; a.dt = dtype; a.b = b; a.t = t; a.d = d;
  a.h0 = h0; a.dzf = dzf; a.dzi = dzi; a.dh0 = dh0;
  a.chunk = chunk;
  a.nchunk = nchunk;
  if (nchunk > 1) {
    const size_t arr = align256((size_t)d * 4 * (size_t)(((int64_t)b * t + 7) / 8));
    uint8_t* p = reinterpret_cast<uint8_t*>(ws);
    a.agg_a = reinterpret_cast<float*>(p);
    a.agg_b = reinterpret_cast<float*>(p + arr);
    a.cin = reinterpret_cast<float*>(p + 2 * arr);
  }
  const size_t es = dsize(dtype);
  const auto aligned = [&](const void* q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) % (2 * es)) == 0; };
  const bool pair = d % 2 == 0 && aligned(zf) && aligned(zi) && aligned(h) && aligned(dh) && aligned(dzf) &&
                    aligned(dzi);
  const int vec = pair ? 2 : 1;
  a.gx = (int32_t)((d / vec + bwd::kScanBwdThreads - 1) / bwd::kScanBwdThreads);
  MMF_CHECK_ARG((int64_t)a.gx * a.nchunk * b < ((int64_t)1 << 31), "scan backward: b * t * d too large for one grid");
  LaunchScope ls(MMF_KERNEL_SCAN, (double)b * t * d * 6.0 * es, st);
  if (a.nchunk > 1) g_launches.fetch_add(2);  // three kernels under one timing scope
  if (dtype == MMF_F32) {
    if (pair) scan_bwd_launch<MMF_F32, 2>(a, st);
    else scan_bwd_launch<MMF_F32, 1>(a, st);
  } else {
    if (pair) scan_bwd_launch<MMF_BF16, 2>(a, st);
    else scan_bwd_launch<MMF_BF16, 1>(a, st);
  }
  return check_launch("scan backward");
}

// ---------------------------------------------------------------------------------------------
// BitLinear training gradients (straight-through estimator)
// ---------------------------------------------------------------------------------------------
mmf_status mmf_bitlinear_backward(const void* x, mmf_dtype x_dtype, int64_t m, const float* norm_w, float eps,
                                  const mmf_ternary* w, const int8_t* q, const float* deq, const void* dy,
                                  mmf_dtype dy_dtype, float* dx, float* dnorm_w, float* dW, void* ws,
                                  size_t ws_bytes, mmf_stream_t stream) {
  MMF_CHECK_ARG(w != nullptr && w->codes && w->scale, "bitlinear backward: null weight");
  MMF_CHECK_ARG(w->n > 0 && w->k > 0 && w->n <= 65535, "bitlinear backward: weight shape [%d][%d]", w->n, w->k);
  MMF_CHECK_ARG(m >= 0 && m <= 0x7fffffff, "bitlinear backward: m = %lld", (long long)m);
  MMF_CHECK_ARG(valid_dtype(x_dtype) && valid_dtype(dy_dtype), "bitlinear backward: bad dtype");
  MMF_CHECK_ARG(m == 0 || (x && q && deq && dy && dx), "bitlinear backward: null pointer");
  const LinBwdPlan plan = lin_bwd_plan(m, w->k, w->n);
  if (m > 0) MMF_TRY(check_ws(ws, ws_bytes, plan.bytes));
  DevInfo* di;
  MMF_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  bwd::LinBwdArgs a;
  memset(&a, 0, sizeof(a));
  a.x = x; a.xdt = x_dtype; a.m = m; a.k = w->k; a.n = w->n; a.norm_w = norm_w; a.eps = eps;
  a.codes = w->codes; a.kw = row_words(w->k); a.scale = w->scale; a.q = q; a.deq = deq;
  a.dy = dy; a.dydt = dy_dtype; a.dx = dx; a.dnorm_w = dnorm_w; a.dW = dW;
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  a.rho = reinterpret_cast<float*>(wsb + plan.rho);
  // dr and dW on the tensor cores unless the CUDA-core engine is forced (mmf_set_gemm_path)
  const bool tc = g_gemm_path.load() != MMF_GEMM_SIMT && di->tc_ready;
  const unsigned kcols = (unsigned)((w->k + bwd::kThreads - 1) / bwd::kThreads);
  LaunchScope ls(MMF_KERNEL_OTHER, (double)m * (w->k * (dsize(x_dtype) + 1.0 + 8.0) + w->n * dsize(dy_dtype)) +
                 (double)w->n * row_words(w->k) * 4.0, st);
  int launches = 0;
  if (m > 0) {
    if (tc) {
      // dr [m][k] = s * dy [m][n] . t [n][k]: A = dy (bf16 as given, else hi / lo rows),
      // B = t transposed to [k][n]
      const bool direct = dy_dtype == MMF_BF16 && w->n % 8 == 0 && aligned16(dy);
      __nv_bfloat16* hi = reinterpret_cast<__nv_bfloat16*>(wsb + plan.dr_hi);
      __nv_bfloat16* lo = reinterpret_cast<__nv_bfloat16*>(wsb + plan.dr_lo);
      __nv_bfloat16* tt = reinterpret_cast<__nv_bfloat16*>(wsb + plan.tt);
      if (!direct) {
        const int64_t total = m * w->n;
        const unsigned blocks = (unsigned)std::min<int64_t>((total + bwd::kThreads - 1) / bwd::kThreads, (int64_t)di->sms * 16);
        launch_k(bwd::lin_bwd_split_kernel, dim3(blocks), dim3(bwd::kThreads), 0, st, a, hi,
                 dy_dtype == MMF_BF16 ? nullptr : lo, plan.ld_n);
        ++launches;
      }
      launch_k(bwd::lin_bwd_transpose_kernel<bwd::kTrTernary>, dim3((unsigned)((w->n + 31) / 32), (unsigned)((w->k + 31) / 32)),
               dim3(32, 8), 0, st, a, tt, nullptr, plan.ld_n);
      ++launches;
      MMF_TRY(launch_bf16_gemm(direct ? dy : hi, direct || dy_dtype == MMF_BF16 ? nullptr : lo,
                               direct ? (int64_t)w->n : plan.ld_n, tt, plan.ld_n, m, w->k, w->n, w->scale, dx, w->k,
                               plan.dr_split, plan.dr_kbc, reinterpret_cast<float*>(wsb + plan.dr_part), st, &launches));
    } else {
      const unsigned words = (unsigned)((w->k + 15) / 16);
      launch_k(bwd::lin_bwd_dr_kernel, dim3((unsigned)m, (words + bwd::kThreads - 1) / bwd::kThreads), dim3(bwd::kThreads),
               0, st, a);
      ++launches;
    }
  }
  if (m > 0) {
    // rho, the gain's gradient partials and dx (in place over dr), one row block per CTA
    float* part = dnorm_w ? reinterpret_cast<float*>(wsb + plan.dnw_part) : nullptr;
    launch_k(bwd::lin_bwd_rows_kernel, dim3((unsigned)plan.dnw_split), dim3(bwd::kThreads), 0, st, a,
             reinterpret_cast<float*>(wsb + plan.mux), part, plan.dnw_rows);
    ++launches;
    if (dnorm_w) {
      launch_k(bwd::lin_bwd_dnw_reduce_kernel, dim3((unsigned)((w->k + 31) / 32)), dim3(32, 8), 0, st, a, part,
               plan.dnw_split);
      ++launches;
    }
  } else if (dnorm_w) {
    cudaError_t e = cudaMemsetAsync(dnorm_w, 0, (size_t)w->k * sizeof(float), st);
    if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
  }
  if (dW && tc && m > 0) {
    // dW [n][k] = (dy (a/127))^T [n][m] . q [m][k]: A = dy scaled and transposed (hi / lo),
    // B = q transposed to [k][m]
    __nv_bfloat16* hi = reinterpret_cast<__nv_bfloat16*>(wsb + plan.dw_hi);
    __nv_bfloat16* lo = reinterpret_cast<__nv_bfloat16*>(wsb + plan.dw_lo);
    __nv_bfloat16* qt = reinterpret_cast<__nv_bfloat16*>(wsb + plan.qt);
    const unsigned rt = (unsigned)((m + 31) / 32);
    launch_k(bwd::lin_bwd_transpose_kernel<bwd::kTrDyScaled>, dim3(rt, (unsigned)((w->n + 31) / 32)), dim3(32, 8), 0, st,
             a, hi, lo, plan.ld_m);
    launch_k(bwd::lin_bwd_transpose_kernel<bwd::kTrCodes>, dim3(rt, (unsigned)((w->k + 31) / 32)), dim3(32, 8), 0, st,
             a, qt, nullptr, plan.ld_m);
    launches += 2;
    MMF_TRY(launch_bf16_gemm(hi, lo, plan.ld_m, qt, plan.ld_m, w->n, w->k, m, nullptr, dW, w->k, plan.dw_split,
                             plan.dw_kbc, reinterpret_cast<float*>(wsb + plan.dw_part), st, &launches));
  } else if (dW) {
    launch_k(bwd::lin_bwd_dw_kernel, dim3(kcols, (unsigned)w->n), dim3(bwd::kThreads), 0, st, a);
    ++launches;
  }
  if (launches > 0) g_launches.fetch_add(launches - 1);  // the timing scope counted one launch itself
  else g_launches.fetch_sub(1);
  return check_launch("bitlinear backward kernels");
}

// ---------------------------------------------------------------------------------------------
// HGRN2 recurrence (state expansion)
// ---------------------------------------------------------------------------------------------
mmf_status mmf_hgrn2_recurrence(const void* q, const void* f, const void* i, mmf_dtype dtype, int32_t b, int64_t t,
                                int32_t heads, int32_t dk, int32_t dv, const float* s0, float* s_out, void* o,
                                mmf_stream_t stream) {
  MMF_CHECK_ARG(b >= 0 && t >= 0 && heads >= 0 && dv >= 0, "hgrn2: negative size");
  MMF_CHECK_ARG(dk >= 1 && dk <= 128, "hgrn2: dk = %d outside [1, 128]", dk);
  MMF_CHECK_ARG(valid_dtype(dtype), "hgrn2: bad dtype");
  MMF_CHECK_ARG(b <= 65535 && heads <= 65535, "hgrn2: b = %d or heads = %d above 65535", b, heads);
  if ((int64_t)b * heads * dv == 0) return MMF_OK;
  MMF_CHECK_ARG(t == 0 || (q && f && i && o), "hgrn2: null pointer");
  DevInfo* di;
  MMF_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  hgrn2::Args a;
  memset(&a, 0, sizeof(a));
  a.q = q; a.f = f; a.i = i; a.dt = dtype; a.b = b; a.t = t; a.heads = heads; a.dk = dk; a.dv = dv;
  a.s0 = s0; a.s_out = s_out; a.o = o;
  const dim3 grid((unsigned)((dv + hgrn2::kCols - 1) / hgrn2::kCols), (unsigned)heads, (unsigned)b);
  const double es = (double)dsize(dtype);
  LaunchScope ls(MMF_KERNEL_OTHER, (double)b * t * heads * (2.0 * dk + 2.0 * dv) * es, st);
#define MMF_HGRN2(DT_, DK_) launch_k(hgrn2::hgrn2_recurrent_kernel<DT_, DK_>, grid, dim3(hgrn2::kThreads), 0, st, a)
  if (dtype == MMF_F32) {
    if (dk <= 16) MMF_HGRN2(MMF_F32, 16);
    else if (dk <= 32) MMF_HGRN2(MMF_F32, 32);
    else if (dk <= 64) MMF_HGRN2(MMF_F32, 64);
    else MMF_HGRN2(MMF_F32, 128);
  } else {
    if (dk <= 16) MMF_HGRN2(MMF_BF16, 16);
    else if (dk <= 32) MMF_HGRN2(MMF_BF16, 32);
    else if (dk <= 64) MMF_HGRN2(MMF_BF16, 64);
    else MMF_HGRN2(MMF_BF16, 128);
  }
#undef MMF_HGRN2
  return check_launch("hgrn2_recurrent_kernel");
}

mmf_status mmf_stack_fwd(const mmf_block_weights* layers, int32_t n_layers, const int32_t* ids,
                         int32_t b, int64_t t, const void* table, int32_t vocab, mmf_dtype dtype,
                         void* y, float* h_last, void* ws, size_t ws_bytes, mmf_stream_t stream) {
  MMF_CHECK_ARG(layers != nullptr && n_layers > 0, "stack: no layers");
  MMF_CHECK_ARG(valid_dtype(dtype), "stack: bad dtype");
  MMF_CHECK_ARG(b >= 0 && t >= 0 && vocab > 0, "stack: bad sizes");
  for (int l = 0; l < n_layers; ++l) {
    MMF_TRY(check_block(&layers[l]));
    MMF_CHECK_ARG(layers[l].d == layers[0].d && layers[l].inner == layers[0].inner,
                  "stack: layer %d has a different shape", l);
  }
  const int64_t m = (int64_t)b * t;
  if (m == 0) return MMF_OK;
  MMF_CHECK_ARG(ids && table && y, "stack: null pointer");
  MMF_CHECK_ARG(aligned16(table) && aligned16(y), "stack: table / y not 16-byte aligned");
  const int32_t d = layers[0].d, inner = layers[0].inner;
  MMF_TRY(check_ws(ws, ws_bytes, mmf_workspace_bytes(MMF_OP_STACK, m, d, inner, n_layers)));
  DevInfo* di;
  MMF_TRY(device_info(&di));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const BlockWs W = block_ws(ws, m, d, inner, dtype);
  uint8_t* pp = reinterpret_cast<uint8_t*>(ws) + W.bytes;
  void* buf[2] = {pp, pp + align256((size_t)m * d * 4)};
  {
    LaunchScope ls(MMF_KERNEL_OTHER, (double)m * d * 2.0 * dsize(dtype) + m * 4.0, st);
    launch_k(embed_gather_kernel, dim3((unsigned)m), dim3(128), 0, st, ids, m, table, dtype, vocab, d, buf[0]);
  }
  MMF_TRY(check_launch("embed_gather_kernel"));
  const void* cur = buf[0];
  for (int l = 0; l < n_layers; ++l) {
    void* out = (l == n_layers - 1) ? y : buf[(l + 1) & 1];
    float* hl = h_last ? h_last + (int64_t)l * b * d : nullptr;
    MMF_TRY(run_block(&layers[l], cur, dtype, b, t, nullptr, out, hl, W, *di, st));
    cur = out;
  }
  return MMF_OK;
}

mmf_status mmf_sync_status(mmf_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  unsigned flag = 0;
  e = cudaMemcpyFromSymbol(&flag, g_device_error, sizeof(flag));
  if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "reading the device error flag: %s", cudaGetErrorString(e));
  if (flag != 0) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return fail(MMF_ERR_CUDA, "clearing the device error flag: %s", cudaGetErrorString(e));
    return fail(MMF_ERR_TIMEOUT, "an in-kernel wait ran out (device flag 0x%x)", flag);
  }
  return MMF_OK;
}

const char* mmf_status_string(mmf_status s) {
  switch (s) {
    case MMF_OK: return "ok";
    case MMF_ERR_INVALID_ARG: return "invalid argument";
    case MMF_ERR_UNSUPPORTED: return "unsupported";
    case MMF_ERR_WORKSPACE: return "workspace too small or misaligned";
    case MMF_ERR_CUDA: return "CUDA error";
    case MMF_ERR_TIMEOUT: return "in-kernel wait timed out";
  }
  return "unknown status";
}

const char* mmf_last_error(void) { return g_last_error.c_str(); }

mmf_status mmf_set_decode_path(mmf_decode_path path) {
  if (path != MMF_DECODE_AUTO && path != MMF_DECODE_FUSED && path != MMF_DECODE_SKINNY && path != MMF_DECODE_BLOCK)
    return fail(MMF_ERR_INVALID_ARG, "bad decode path %d", (int)path);
  g_decode_path.store(path);
  return MMF_OK;
}

int32_t mmf_decode_path_for(int32_t b, int32_t d, int32_t inner) {
  if (b <= 0 || d <= 0 || inner <= 0) return -1;
  return decode_path_for(b, d, inner) == kDecFused ? MMF_DECODE_FUSED
         : decode_path_for(b, d, inner) == kDecSkinny ? MMF_DECODE_SKINNY : MMF_DECODE_BLOCK;
}

mmf_status mmf_set_gemm_path(mmf_gemm_path path) {
  if (path != MMF_GEMM_AUTO && path != MMF_GEMM_TENSOR && path != MMF_GEMM_SIMT)
    return fail(MMF_ERR_INVALID_ARG, "bad gemm path %d", (int)path);
  g_gemm_path.store(path);
  return MMF_OK;
}

uint64_t mmf_launch_count(void) { return g_launches.load(); }

mmf_status mmf_timing_enable(int on) {
  g_timing.store(on ? 1 : 0);
  return MMF_OK;
}

mmf_status mmf_timing_read(mmf_kernel_class cls, int64_t* launches, double* total_ms, double* work) {
  if ((int)cls < 0 || (int)cls >= MMF_KERNEL_CLASSES) return fail(MMF_ERR_INVALID_ARG, "bad kernel class %d", (int)cls);
  std::lock_guard<std::mutex> lk(g_tmu);
  int64_t n = 0;
  double ms = 0.0, wk = 0.0;
  std::vector<TimedRec> keep;
  mmf_status st = MMF_OK;
  for (const TimedRec& r : g_recs) {
    if (r.cls != (int)cls) {
      keep.push_back(r);
      continue;
    }
    float e = 0.0f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&e, r.a, r.b) != cudaSuccess)
      st = fail(MMF_ERR_CUDA, "timing events failed");
    ms += e;
    wk += r.work;
    ++n;
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_recs.swap(keep);
  if (launches) *launches = n;
  if (total_ms) *total_ms = ms;
  if (work) *work = wk;
  return st;
}

mmf_status mmf_set_wait_limit(uint32_t microseconds) {
  g_wait_limit.store(microseconds == 0 ? kDefaultWaitLimit : microseconds);
  return MMF_OK;
}

}  // extern "C"
