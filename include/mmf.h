/*
 * mmf.h -- C ABI of the B200 (sm_100a) HGRNBit block forward library (libmmf.so).
 *
 * What it computes. The MatMul-free language model replaces every dense projection with a
 * FusedBitLinear and replaces attention with a gated linear recurrence:
 *   - FusedBitLinear: RMSNorm (eps 1e-08), per-token absmax INT8 activation quantisation,
 *     ternary {-1, 0, +1} weights by round-to-nearest of W / mean|W|, an exact integer product
 *     and a rescale.  Sources: nightvoyager.top "MatMul-Free LLM" report, innovations table
 *     (ternary weight_quant) and reusable-patterns list (RMSNorm fused with INT8 quantisation);
 *     hysenlabs.com, "HGRNBitBlock structure" (i/f/g/o_proj, gate_proj, down_proj are each a
 *     FusedBitLinear with an RMSNorm of eps=1e-08).
 *   - HGRN recurrence h_t = f_t * h_{t-1} + i_t per channel, O(T*D) (nightvoyager.top, innovations
 *     table), closed by g_norm = RMSNorm(h) * SiLU(g) (FusedRMSNormSwishGate, hysenlabs.com block
 *     structure) and an MLP gate_proj -> SiLU gate -> down_proj whose gate_proj is twice as wide
 *     as down_proj's input (11264 vs 5632 at hidden 2048, same section).
 *
 * Conventions shared by every call.
 *   Memory:   every pointer argument is DEVICE memory unless its comment says host. The caller
 *             owns all buffers and streams; the library allocates nothing. Calls that need
 *             scratch take a caller buffer `ws` of at least mmf_workspace_bytes(...) bytes,
 *             aligned to 256 bytes, which must not be used by anything else until the stream has
 *             passed the call.
 *   Streams:  every compute call only enqueues work on `stream` (0 = legacy default stream) and
 *             returns before it runs.
 *   Layouts:  activations are row-major [rows][features]; weights follow PyTorch's Linear layout
 *             [out_features N][in_features K], y = x W^T.
 *   Dtypes:   MMF_F32 or MMF_BF16 for activations; reductions, the recurrence and epilogues run in
 *             float32 whatever the storage type; integer products are exact int32.
 *   Errors:   arguments are validated on the host before anything is enqueued; a bad argument
 *             returns MMF_ERR_INVALID_ARG (or MMF_ERR_UNSUPPORTED / MMF_ERR_WORKSPACE) and enqueues
 *             nothing. A failed launch returns MMF_ERR_CUDA. Every wait inside a kernel is bounded:
 *             when one runs out the kernel records MMF_ERR_TIMEOUT in a device flag, drains its own
 *             in-flight copies, releases its tensor memory and returns; mmf_sync_status() reports
 *             and clears that flag. There is no fallback path: an unsupported case is an error.
 *             mmf_last_error() gives a one-line description of the last failure on this thread.
 *   Alignment: device pointers must be 16-byte aligned.
 *
 * Packed ternary format (this library's own; the pages fix only "ternary codes plus a scale").
 *   One weight matrix [N][K] is stored as u32 words codes[N][mmf_packed_row_words(K)] plus one
 *   float32 scale s = max(mean|W|, 1e-5). A row holds 16 codes per word and is padded with zero
 *   codes to a multiple of 64 codes, so every row starts on a 16-byte boundary. Column
 *   k = 16*w + 4*quad + lane (quad, lane in 0..3) sits in word w at bit
 *   16*(quad >> 1) + 2*(quad & 1) + 4*lane as a two's-complement 2-bit field: 00 = 0, 01 = +1,
 *   11 = -1 (10 is never written). This puts the four codes of one quad in the low two bits of
 *   the four nibbles of one 16-bit half, so a byte permute expands four codes to four int8 lanes.
 */
#ifndef MMF_H_
#define MMF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mmf_stream_t; /* a cudaStream_t */

typedef enum {
  MMF_OK = 0,
  MMF_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size or dtype */
  MMF_ERR_UNSUPPORTED = 2, /* valid request the library cannot serve (e.g. no sm_100a device) */
  MMF_ERR_WORKSPACE = 3,   /* ws smaller than mmf_workspace_bytes() or misaligned */
  MMF_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  MMF_ERR_TIMEOUT = 5      /* a bounded in-kernel wait ran out (reported by mmf_sync_status) */
} mmf_status;

typedef enum { MMF_F32 = 0, MMF_BF16 = 1 } mmf_dtype;

/* Workspace queries: which call the scratch is for. */
typedef enum {
  MMF_OP_PACK = 0,      /* mmf_pack_ternary: m = n*k elements                     */
  MMF_OP_BITLINEAR = 1, /* mmf_bitlinear_fwd: m rows, d = K, inner = N            */
  MMF_OP_BLOCK = 2,     /* mmf_block_fwd: m = b*t tokens, d, inner                */
  MMF_OP_DECODE = 3,    /* mmf_decode_step: m = b, d, inner                       */
  MMF_OP_STACK = 4,     /* mmf_stack_fwd: m = b*t tokens, d, inner, n_layers      */
  MMF_OP_SCAN = 5,      /* mmf_hgrn_scan: m = b*t tokens, d channels              */
  MMF_OP_HEAD = 6,      /* mmf_lm_head_argmax: inner = vocabulary size            */
  MMF_OP_BITLINEAR_BWD = 7 /* mmf_bitlinear_backward: m rows, d = K, inner = N     */
} mmf_op;

/* A packed ternary weight (device pointers). */
typedef struct {
  const uint32_t* codes; /* [n][mmf_packed_row_words(k)] u32, format above */
  const float* scale;    /* 1 float: s = max(mean|W|, 1e-5)                   */
  int32_t n;             /* out_features */
  int32_t k;             /* in_features  */
} mmf_ternary;

/* One HGRNBit block (hysenlabs.com block structure). Gains are device float32 vectors:
 * nw_i/f/g/o/gate have d entries, nw_down has `inner`, gnorm_w has d. The GLU reading:
 * gate_proj rows [0, inner) are the SiLU gate, rows [inner, 2*inner) the linear "up" half. */
typedef struct {
  int32_t d;     /* hidden size, 1 to 32768 */
  int32_t inner; /* MLP inner size I, 1 to 32768; gate_proj is [2I][d], down_proj is [d][I] */
  float eps;     /* RMSNorm eps of every norm in the block (1e-8), >= 0 */
  const float *nw_i, *nw_f, *nw_g, *nw_o, *nw_gate, *nw_down, *gnorm_w;
  mmf_ternary i, f, g, o, gate, down;
} mmf_block_weights;

/* ---- sizes ---------------------------------------------------------------------------------- */

/* u32 words in one packed row of k codes: 4 * ceil(k / 64). */
int32_t mmf_packed_row_words(int32_t k);
/* u32 words of a packed [n][k] matrix: n * mmf_packed_row_words(k). */
size_t mmf_packed_words(int32_t n, int32_t k);
/* Scratch bytes that `op` needs for the given sizes (0 if none). */
size_t mmf_workspace_bytes(mmf_op op, int64_t m, int32_t d, int32_t inner, int32_t n_layers);

/* ---- calls ---------------------------------------------------------------------------------- */

/* Ternarise and pack one weight matrix (weight_quant, nightvoyager.top innovations table:
 * round-to-nearest onto {-1, 0, +1}).
 *   w          [n][k] MMF_F32 or MMF_BF16 latent weights.
 *   codes_out  [n][mmf_packed_row_words(k)] u32, written entirely (padding codes are 0).
 *   scale_out  1 float: s = max(mean|W|, 1e-5), with mean|W| summed in float64.
 *   Codes are t = clamp(rint(w / s), -1, 1) with the division in float32 (IEEE, ties to even).
 *   ws >= mmf_workspace_bytes(MMF_OP_PACK, n*k, 0, 0, 0). Deterministic. */
mmf_status mmf_pack_ternary(const void* w, mmf_dtype w_dtype, int32_t n, int32_t k,
                            uint32_t* codes_out, float* scale_out, void* ws, size_t ws_bytes,
                            mmf_stream_t stream);

/* One FusedBitLinear, y = BitLinear(x) (nightvoyager.top reusable patterns; hysenlabs.com block
 * structure):
 *   r = x / sqrt(mean(x^2) + eps) * norm_w              (eps = 1e-8)
 *   a = max(max|r|, 1e-5);  q = clamp(rint(r * (127/a)), -127, 127)   (int8, float32 decision)
 *   acc[m][n] = sum_k q[m][k] * t[n][k]                 (exact int32)
 *   y[m][n] = acc * (a/127) * s
 *   x       [m][w->k] x_dtype, 16-byte aligned.    norm_w [w->k] float32, or NULL for a unit gain.
 *   y       [m][w->n] y_dtype, 16-byte aligned.
 *   w       1 <= w->k <= 32768, w->n >= 1; codes 16-byte aligned, codes and scale non-NULL.
 *   q_dbg   optional [m][w->k] int8: the activation codes.
 *   deq_dbg optional [m] float32: a/127 per row.
 *   acc_dbg optional [m][w->n] int32: the integer accumulators.
 *   ws >= mmf_workspace_bytes(MMF_OP_BITLINEAR, m, w->k, w->n, 0).  m = 0 is a no-op. */
mmf_status mmf_bitlinear_fwd(const void* x, mmf_dtype x_dtype, int64_t m, const float* norm_w,
                             const mmf_ternary* w, void* y, mmf_dtype y_dtype, int8_t* q_dbg,
                             float* deq_dbg, int32_t* acc_dbg, void* ws, size_t ws_bytes,
                             mmf_stream_t stream);

/* HGRN gated linear recurrence with its gates fused in (nightvoyager.top innovations table):
 *   f = sigmoid(zf);  i = SiLU(zi) * (1 - f);  h_t = f_t * h_{t-1} + i_t,  h_{-1} = h0 or 0.
 *   zf, zi  [b][t][z_stride] z_dtype, channels [0, d) of each row are used (z_stride >= d).
 *   h0      optional [b][d] float32 (may alias h_last: read before it is written).
 *   h_out   [b][t][d] h_dtype.   h_last optional [b][d] float32 (= h at the last step).
 *   ws >= mmf_workspace_bytes(MMF_OP_SCAN, b*t, d, 0, 0) when t > 16 (unused otherwise).
 *   Chunked: per (channel, chunk of steps) affine aggregates, a carry pass per channel, then a
 *   replay that stores h; float32 carries throughout. */
mmf_status mmf_hgrn_scan(const void* zf, const void* zi, mmf_dtype z_dtype, int64_t z_stride,
                         int32_t b, int64_t t, int32_t d, const float* h0, void* h_out,
                         mmf_dtype h_dtype, float* h_last, void* ws, size_t ws_bytes,
                         mmf_stream_t stream);

/* One HGRNBit block forward over b sequences of t tokens (hysenlabs.com block structure):
 *   zi, zf, g = i/f/g_proj(x);  h = scan(f = sigmoid(zf), i = SiLU(zi)(1-f));
 *   u = RMSNorm(h) * gnorm_w * SiLU(g);  x1 = x + o_proj(u);
 *   [a | c] = gate_proj(x1);  y = x1 + down_proj(SiLU(a) * c).
 *   x, y    [b][t][d] dtype (may not alias).   h0 optional [b][d] float32 initial state.
 *   h_last  optional [b][d] float32 final state.
 *   ws >= mmf_workspace_bytes(MMF_OP_BLOCK, b*t, d, inner, 1). */
mmf_status mmf_block_fwd(const mmf_block_weights* w, const void* x, mmf_dtype dtype, int32_t b,
                         int64_t t, const float* h0, void* y, float* h_last, void* ws,
                         size_t ws_bytes, mmf_stream_t stream);

/* Debug taps of one block forward: every non-NULL pointer receives a copy of that intermediate,
 * taken after the forward from the very buffers its kernels used (m = b*t tokens, es = dtype):
 *   q_ifg [3][m][d] int8 and deq_ifg [3][m] float: activation codes / a/127 of the i, f, g inputs
 *   z [m][3d] dtype = [zi | zf | g];  h [m][d] dtype;  q_o [m][d], deq_o [m]: o_proj input codes
 *   x1 [m][d] dtype;  q_gate [m][d], deq_gate [m]
 *   gu [m][2I] dtype = [gate | up], written when gate_proj stores both halves;
 *   v [m][I] dtype = SiLU(gate) * up, written instead when gate_proj's epilogue forms the GLU
 *     product itself: on the tensor-core engine (8 or more rows under MMF_GEMM_AUTO, or
 *     MMF_GEMM_TENSOR) with I % 64 == 0
 *   q_down [m][I], deq_down [m]. */
typedef struct {
  int8_t* q_ifg;
  float* deq_ifg;
  void* z;
  void* h;
  int8_t* q_o;
  float* deq_o;
  void* x1;
  int8_t* q_gate;
  float* deq_gate;
  void* gu;
  int8_t* q_down;
  float* deq_down;
  void* v;
} mmf_block_taps;

/* mmf_block_fwd followed by copies of its intermediates into `taps` (same kernels, same
 * workspace). For tests and debugging; the copies add traffic. */
mmf_status mmf_block_fwd_taps(const mmf_block_weights* w, const void* x, mmf_dtype dtype, int32_t b,
                              int64_t t, const float* h0, void* y, float* h_last,
                              const mmf_block_taps* taps, void* ws, size_t ws_bytes,
                              mmf_stream_t stream);

/* One autoregressive step through n_layers blocks: the block above with t = 1 and the
 * recurrent state carried per layer.
 *   layers  HOST array of n_layers block descriptors (device pointers inside).
 *   x       [b][d] dtype: hidden state of the current token entering layer 0.
 *   state   [n_layers][b][d] float32, read and overwritten in place.
 *   y       [b][d] dtype: hidden state leaving the last layer (may not alias x).
 *   ws >= mmf_workspace_bytes(MMF_OP_DECODE, b, d, inner, n_layers).
 * Which kernels run is set by mmf_set_decode_path (below): four fused CUDA-core launches per
 * block, four skinny tensor-core products each followed by a row stage, or the block path with
 * t = 1. Same arithmetic either way. */
mmf_status mmf_decode_step(const mmf_block_weights* layers, int32_t n_layers, const void* x,
                           mmf_dtype dtype, int32_t b, float* state, void* y, void* ws,
                           size_t ws_bytes, mmf_stream_t stream);

/* Debug taps of one decode step, one struct per layer; every non-NULL pointer receives that
 * intermediate of the layer (b token rows, es = dtype):
 *   q_ifg [3][b][d] int8, deq_ifg [3][b]: codes / a/127 of the i, f, g inputs
 *   z [b][3d] float32 = [zi | zf | g]      h [b][d] float32: the h that g_norm reads
 *   q_o [b][d], deq_o [b]                  x1 [b][d] dtype
 *   q_gate [b][d], deq_gate [b]
 *   v [b][I] dtype = SiLU(gate) * up, written when the step forms it (the fused decode, or the
 *     block path with the GLU in gate_proj's epilogue); gu [b][2I] dtype = [gate | up] otherwise
 *   q_down [b][I], deq_down [b]            y [b][d] dtype: the layer's output
 * On the block path z and h are the stored dtype values widened to float32. */
typedef struct {
  int8_t* q_ifg;
  float* deq_ifg;
  float* z;
  float* h;
  int8_t* q_o;
  float* deq_o;
  void* x1;
  int8_t* q_gate;
  float* deq_gate;
  void* gu;
  void* v;
  int8_t* q_down;
  float* deq_down;
  void* y;
} mmf_decode_taps;

/* mmf_decode_step with the intermediates of every layer copied into taps[0 .. n_layers) (HOST
 * array): same kernels and workspace; for tests and debugging (the copies add traffic). */
mmf_status mmf_decode_step_taps(const mmf_block_weights* layers, int32_t n_layers, const void* x,
                                mmf_dtype dtype, int32_t b, float* state, void* y,
                                const mmf_decode_taps* taps, void* ws, size_t ws_bytes,
                                mmf_stream_t stream);

/* Token embedding gather: out[r] = table[ids[r]] for r < m.
 *   ids [m] int32. Ids live on the device and are not checked on the host; an id outside
 *   [0, vocab) yields a zero row (never an out-of-bounds read).
 *   table [vocab][d] dtype; out [m][d] dtype. */
mmf_status mmf_embed_gather(const int32_t* ids, int64_t m, const void* table, mmf_dtype dtype,
                            int32_t vocab, int32_t d, void* out, mmf_stream_t stream);

/* Tied language-model head and greedy next token, for generation: only the last position of
 * each sequence is needed, so x holds one row per sequence.
 *   logits[r][v] = sum_k RMSNorm(x[r])[k] * table[v][k], RMSNorm(x) = x / sqrt(mean(x^2) + eps)
 *   * norm_w (the final norm after the last block); ids[r] = argmax_v logits[r][v], the lowest
 *   index among equal maxima (greedy decoding).
 * Readings: the head shares the embedding table (tied); the final norm has the blocks' eps
 * (hysenlabs.com "MatMul-Free LM", install and model-table sections: 32000-word vocabulary,
 * causal-LM generation example).
 *   x       [b][d] x_dtype, 16-byte aligned; d a multiple of 8, d * 4 <= 200 KB.
 *   norm_w  [d] float32 or NULL (= 1).
 *   table   [vocab][d] table_dtype (the embedding table), 16-byte aligned.
 *   ids     [b] int32 out.   logits [b][vocab] float32 out or NULL (a test tap).
 *   ws >= mmf_workspace_bytes(MMF_OP_HEAD, 0, d, vocab, 0); a smaller ws is an error.
 * bf16 table and b >= 2: tensor cores (tcgen05, bf16 operands, float32 accumulation); each
 * normalised row enters as a bf16 pair hi + lo (16 significant bits), the table streams once per
 * 128 rows. Otherwise CUDA cores, float32 accumulation, the table streamed once per 8 rows. */
mmf_status mmf_lm_head_argmax(const void* x, mmf_dtype x_dtype, int32_t b, int32_t d, const float* norm_w,
                              float eps, const void* table, mmf_dtype table_dtype, int32_t vocab,
                              int32_t* ids, float* logits, void* ws, size_t ws_bytes, mmf_stream_t stream);

/* Integrity check of a packed ternary matrix (the format above): *bad (device, 8-byte aligned)
 * receives the number of malformed 2-bit fields: fields of real columns holding the unused
 * pattern 10, plus nonzero fields in each row's padding columns k .. 16 * mmf_packed_row_words(k)
 * - 1 (each field counts once); 0 means the codes are well formed. w->codes 16-byte aligned. The
 * count is reset and written on `stream` (read it after mmf_sync_status). Any shape. */
mmf_status mmf_validate_packed(const mmf_ternary* w, unsigned long long* bad, mmf_stream_t stream);

/* Training gradients of FusedBitLinear with the straight-through estimator (nightvoyager.top,
 * innovations table: weight_quant quantises in the forward pass and keeps the gradient in the
 * backward pass; the activation quantiser is read the same way). With the forward's activation
 * codes q and factors a/127 (mmf_bitlinear_fwd's q_dbg and deq_dbg), rq = q (a/127), Wq = t s:
 *   dr = dy Wq;  u = dr norm_w;  rho = (mean(x^2) + eps)^(-1/2)
 *   dx = rho u - rho^3 x mean(u x)                     [m][w->k] float32 out
 *   dnorm_w[k] = sum_m dr[m][k] x[m][k] rho_m          [w->k] float32 out, or NULL
 *   dW = dy^T rq (the latent float weight's gradient)  [w->n][w->k] float32 out, or NULL
 *   x [m][w->k] x_dtype; norm_w [w->k] float32 or NULL (unit gain); q [m][w->k] int8;
 *   deq [m] float32; dy [m][w->n] dy_dtype. w->n <= 65535; 0 <= m <= 2^31 - 1.
 *   ws >= mmf_workspace_bytes(MMF_OP_BITLINEAR_BWD, m, w->k, w->n, 0), 256-byte aligned,
 *   caller-owned. m = 0 writes zero dnorm_w / dW.
 * dr and dW run on the bf16 tensor cores (tcgen05.mma.kind::f16, float32 accumulation): dy (and
 * dy (a/127) for dW) enters as bf16 hi / lo pairs, the ternary and int8 codes are exact in bf16,
 * so both products are float32-accurate (about 2^-17 relative per term); the operands are first
 * laid out K-major in the workspace (transposes of t, q and dy). mmf_set_gemm_path(MMF_GEMM_SIMT)
 * selects CUDA-core kernels with float32 arithmetic instead. rho, the gain's gradient and dx are
 * CUDA-core kernels either way. */
mmf_status mmf_bitlinear_backward(const void* x, mmf_dtype x_dtype, int64_t m, const float* norm_w, float eps,
                                  const mmf_ternary* w, const int8_t* q, const float* deq, const void* dy,
                                  mmf_dtype dy_dtype, float* dx, float* dnorm_w, float* dW, void* ws,
                                  size_t ws_bytes, mmf_stream_t stream);

/* Gradients of mmf_hgrn_scan for a training step (the recurrence and its gates are smooth, so
 * these are exact derivatives; nightvoyager.top, innovations table, names the training method):
 *   forward  f = sigmoid(zf), i = SiLU(zi) (1 - f), h_t = f_t h_{t-1} + i_t, h_{-1} = h0 or 0;
 *   G_t = dh_t + f_{t+1} G_{t+1} (backwards in time), di_t = G_t, df_t = G_t h_{t-1};
 *   dzf = (df - di SiLU(zi)) f (1 - f);  dzi = di (1 - f) SiLU'(zi);  dh0 = f_0 G_0.
 *   zf, zi, h (the forward's states), dh (dL/dh) [b][t][d] dtype, contiguous.
 *   h0 [b][d] float32 or NULL.   dzf, dzi [b][t][d] dtype out.   dh0 [b][d] float32 out or NULL.
 *   ws >= mmf_workspace_bytes(MMF_OP_SCAN, b*t, d, 0, 0) when t > 32 (unused otherwise), 256-byte
 *   aligned, caller-owned, not retained; a smaller or misaligned ws is MMF_ERR_WORKSPACE.
 *   t = 0 writes dh0 = 0. Chunks of 32 steps up to t = 4096, else at most 128 chunks; b x chunks x
 *   ceil(d / 256) CTAs (ceil(d / 128) for odd d or rows not 2-element aligned) must be < 2^31.
 * CUDA cores, float32 arithmetic, chunked like the forward scan with time reversed: G is affine
 * in the carry from the later steps, so chunks fold to (A, B), a reverse walk over the chunks
 * gives each its carry, and each chunk is replayed from it. The chunk sums associate differently
 * from one sequential reverse walk (float32 rounding order only). */
mmf_status mmf_hgrn_scan_backward(const void* zf, const void* zi, const void* h, const void* dh, mmf_dtype dtype,
                                  int32_t b, int64_t t, int32_t d, const float* h0, void* dzf, void* dzi,
                                  float* dh0, void* ws, size_t ws_bytes, mmf_stream_t stream);

/* HGRN2 recurrence with state expansion, per sequence and head (nightvoyager.top, innovations
 * table, names HGRN2 and its fused-recurrent and chunked kernels; the recurrence is HGRN2's
 * published one, the pages print no equations):
 *   S_t = diag(f_t) S_{t-1} + (1 - f_t)^T i_t   (S_t: dk x dv, S_{-1} = s0 or 0)
 *   o_t = q_t S_t
 *   q, f  [b][t][heads][dk] dtype, contiguous; f are forget gates in [0, 1] (gating applied by
 *         the caller).   i [b][t][heads][dv] dtype.   o [b][t][heads][dv] dtype out.
 *   s0    [b][heads][dk][dv] float32 or NULL (zeros).   s_out same shape float32 out, or NULL.
 *   1 <= dk <= 128; b, heads <= 65535. t = 0 writes only s_out.
 * CUDA cores, float32 state and accumulation: four threads per (sequence, head, value column),
 * each holding a quarter of the column's state rows, steps in order. No workspace. */
mmf_status mmf_hgrn2_recurrence(const void* q, const void* f, const void* i, mmf_dtype dtype, int32_t b, int64_t t,
                                int32_t heads, int32_t dk, int32_t dv, const float* s0, float* s_out, void* o,
                                mmf_stream_t stream);

/* Prefill forward of an HGRNBitModel block stack (hysenlabs.com: HGRNBitModel = embedding + a
 * stack of HGRNBitBlock): embedding gather, then the n_layers blocks in order.
 *   layers  HOST array of n_layers block descriptors.  ids [b][t] int32.
 *   table   [vocab][d] dtype.   y [b][t][d] dtype.
 *   h_last  optional [n_layers][b][d] float32 final recurrent state of every layer.
 *   ws >= mmf_workspace_bytes(MMF_OP_STACK, b*t, d, inner, n_layers). */
mmf_status mmf_stack_fwd(const mmf_block_weights* layers, int32_t n_layers, const int32_t* ids,
                         int32_t b, int64_t t, const void* table, int32_t vocab, mmf_dtype dtype,
                         void* y, float* h_last, void* ws, size_t ws_bytes, mmf_stream_t stream);

/* ---- allocation-free variant (no counterpart on the pages) ---------------------------------- */

/* Bytes of the library's static scratch array used by mmf_bitlinear_fwd_noalloc (8 MiB). */
#define MMF_NOALLOC_SCRATCH_BYTES (8u << 20)

/* mmf_bitlinear_fwd for callers that cannot allocate device memory and have no workspace to pass:
 * a plug-in or custom-op interface that hands an operation only its input and output buffers,
 * a host runtime that has reserved all device memory for its own pool, or a latency-critical
 * loop where cudaMalloc / cudaFree (which can synchronise the device) are not allowed. It computes
 * exactly what mmf_bitlinear_fwd computes (same kernels; no debug taps) and calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *   Scratch: the int8 activation codes and per-row factors live in one file-scope device array of
 *   MMF_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the library holds until the
 *   process exits. A call needs mmf_workspace_bytes(MMF_OP_BITLINEAR, m, w->k, w->n, 0) bytes of
 *   it; larger requests return MMF_ERR_WORKSPACE before anything is enqueued.
 *   Set-up: the first call on each device looks up the array's device address on that device
 *   (the device must be current); make that first call before any stream capture begins. The
 *   address belongs to the device's context: after a cudaDeviceReset the next call looks it up
 *   again (that call, too, should come before any stream capture).
 *   Sharing: every call on a device uses the same array and leaves its contents behind; the
 *   kernels overwrite every byte they read, so nothing needs clearing between calls. Calls whose
 *   execution overlaps on the GPU (other streams, other host threads) race on the array: order
 *   them on one stream or synchronise between them. */
mmf_status mmf_bitlinear_fwd_noalloc(const void* x, mmf_dtype x_dtype, int64_t m, const float* norm_w,
                                     const mmf_ternary* w, void* y, mmf_dtype y_dtype,
                                     mmf_stream_t stream);

/* ---- status, errors and tuning --------------------------------------------------------------- */

/* Synchronise `stream`, then report and clear the device error flag: MMF_OK,
 * MMF_ERR_TIMEOUT (an in-kernel wait ran out) or MMF_ERR_CUDA (the stream reported an error). */
mmf_status mmf_sync_status(mmf_stream_t stream);
/* Static description of a status code. */
const char* mmf_status_string(mmf_status s);
/* Description of the last failure on the calling thread ("" if none). */
const char* mmf_last_error(void);

/* Which integer-product engine the BitLinear calls use (process-wide, not thread-safe):
 *   MMF_GEMM_AUTO   tensor-core kernel (tcgen05 int8 MMA, TMEM accumulators) for row counts
 *                   where it pays, CUDA-core kernel otherwise (default);
 *   MMF_GEMM_TENSOR always the tensor-core kernel;
 *   MMF_GEMM_SIMT   always the CUDA-core kernel.
 * Both produce identical int32 accumulators; tests use this to check each on every shape. */
typedef enum { MMF_GEMM_AUTO = 0, MMF_GEMM_TENSOR = 1, MMF_GEMM_SIMT = 2 } mmf_gemm_path;
mmf_status mmf_set_gemm_path(mmf_gemm_path path);

/* Which kernels a decode step (mmf_decode_step) runs (process-wide, not thread-safe):
 *   MMF_DECODE_AUTO    the fused CUDA-core path for 1 or 2 rows, the skinny tensor-core path
 *                      for 3 to 64 rows, the block path above (default); with the CUDA-core engine
 *                      (mmf_set_gemm_path) the fused path for 1, 2, 4 or 8 rows and the block path
 *                      otherwise; with the tensor-core engine the block path;
 *   MMF_DECODE_FUSED   four fused CUDA-core launches per block (1, 2, 4 or 8 rows, d and inner
 *                      multiples of 8; other counts take the block path);
 *   MMF_DECODE_SKINNY  per block four skinny tensor-core products into exact int32 accumulators
 *                      (narrow token tiles of 16 / 32 / 64, K split across a thread-block cluster
 *                      and reduced through distributed shared memory), each followed by a row
 *                      stage that applies the product's epilogue and quantises the next input
 *                      (1 to 64 rows, d and inner multiples of 8 up to 8192, 16-byte aligned
 *                      norm gains; otherwise the block path);
 *   MMF_DECODE_BLOCK   the prefill block forward with t = 1 (norm-quant, GEMM, scan kernels).
 * All paths compute the same arithmetic; tests use this to check each. */
typedef enum { MMF_DECODE_AUTO = 0, MMF_DECODE_FUSED = 1, MMF_DECODE_SKINNY = 2, MMF_DECODE_BLOCK = 3 } mmf_decode_path;
mmf_status mmf_set_decode_path(mmf_decode_path path);
/* The path (MMF_DECODE_FUSED / SKINNY / BLOCK) a decode step of b rows takes under the current
 * settings, or -1 for sizes that are not positive. */
int32_t mmf_decode_path_for(int32_t b, int32_t d, int32_t inner);

/* Wall-clock cap, in microseconds, of every bounded in-kernel wait (default 2,000,000 = 2 s;
 * 0 restores the default), measured on the GPU's global timer. Lowering it makes waits run out
 * early, which the fault tests use to exercise the timeout path without hanging or faulting the
 * GPU. Process-wide; read at launch. */
mmf_status mmf_set_wait_limit(uint32_t microseconds);

/* ---- instrumentation (benchmarks; no counterpart on the pages) ------------------------------ */

typedef enum {
  MMF_KERNEL_GEMM_TC = 0,    /* tensor-core ternary GEMM; work = integer ops 2*m*n*k          */
  MMF_KERNEL_GEMM_SIMT = 1,  /* CUDA-core ternary GEMM; work = algorithmic HBM bytes            */
  MMF_KERNEL_NORM_QUANT = 2, /* RMSNorm + int8 quant (+GLU / g_norm); work = HBM bytes          */
  MMF_KERNEL_SCAN = 3,       /* HGRN scan; work = HBM bytes                                       */
  MMF_KERNEL_OTHER = 4,      /* pack, embedding gather; work = HBM bytes                          */
  MMF_KERNEL_CLASSES = 5
} mmf_kernel_class;

/* Kernels launched by this process through the library so far. */
uint64_t mmf_launch_count(void);
/* When on (process-wide), every launch is bracketed by two CUDA events recorded on the launch's
 * own stream. Leave it off while a stream is being captured into a CUDA graph. */
mmf_status mmf_timing_enable(int on);
/* Synchronise on the recorded events and return, for kernel class `cls`, the launches, their
 * total device milliseconds and their total algorithmic work (see mmf_kernel_class) recorded
 * since the previous read of that class; the class's records are then cleared. */
mmf_status mmf_timing_read(mmf_kernel_class cls, int64_t* launches, double* total_ms, double* work);

#ifdef __cplusplus
}
#endif
#endif /* MMF_H_ */
