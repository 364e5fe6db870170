/*
 * ccgqa.h -- C ABI of the B200 (sm_100a) CCGQA forward hot path.
 *
 * CCGQA (Compressed Convolutional Grouped-Query Attention) runs causal softmax
 * attention entirely inside a latent space of width E / C:
 *   "Compressed Convolutional Attention: Efficient Attention in a Compressed
 *   Latent Space", section "Methodologie" items 1-4 (latent projection,
 *   convolutional mixing with QK-mean, value-shift, RoPE in the latent heads)
 *   and section "Compressed Convolutional Grouped Query Attention (CCGQA)"
 *   (kv heads shared by groups of query heads, as in "Grouped Query Attention
 *   (GQA)", section "Cómo funciona GQA").
 *
 * Geometry: d = E / (C * n_q_heads) is the head dim, G = n_q_heads / n_kv_heads
 * the group size; query head h reads kv head h / G.  N_qkv = (Hq + 2 Hkv) d.
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers, row-major, densely packed, owned
 *    by the caller; the library allocates no memory and keeps no state beyond
 *    a launch counter, the last CUDA error of each thread, the optional
 *    per-thread timing hook, the process-wide fused-projection switch and the
 *    allocation-free decode entry point's scratch array (all below), and a
 *    record of the kernels whose shared-memory limit it has already raised.
 *    Element type is cfg->dtype (fp32 or bf16)
 *    unless stated.  Every pointer must be 16-byte aligned.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream).  Host-side validation happens first: on any
 *    invalid argument the call returns an error status and launches nothing.
 *  - `dev_err` (nullable) is a device int32 that kernels OR error bits into
 *    (CCGQA_DEVERR_*); the library never clears it.  A kernel that detects an
 *    out-of-range index or capacity overflow skips the access and sets a bit;
 *    no kernel traps.  Every wait inside a kernel is bounded; a wait that runs
 *    out sets CCGQA_DEVERR_TIMEOUT and the kernel returns (outputs invalid).
 *  - Returns CCGQA_ERR_CUDA when a launch fails (cudaGetLastError).
 */
#ifndef CCGQA_H
#define CCGQA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CCGQA_API __attribute__((visibility("default")))

typedef enum {
  CCGQA_OK = 0,
  CCGQA_ERR_INVALID_ARG = 1,  /* NULL / misaligned pointer, inconsistent sizes */
  CCGQA_ERR_UNSUPPORTED = 2,  /* valid but not implemented: d outside {16, 32, 64,
                                 128}, or a group so large that (G + 2) d channels of
                                 one sequence do not fit the decode pre-step's
                                 shared memory */
  CCGQA_ERR_CAPACITY = 3,     /* the tokens do not fit the cache capacity */
  CCGQA_ERR_WORKSPACE = 4,    /* workspace NULL, misaligned or too small */
  CCGQA_ERR_CUDA = 5          /* a CUDA runtime call or launch failed */
} ccgqa_status;

typedef enum { CCGQA_F32 = 0, CCGQA_BF16 = 1 } ccgqa_dtype;

/* Device-side error bits OR-ed into *dev_err. */
#define CCGQA_DEVERR_INDEX 1     /* an index fell outside its buffer; access skipped */
#define CCGQA_DEVERR_TIMEOUT 2   /* a bounded in-kernel wait ran out */
#define CCGQA_DEVERR_CAPACITY 4  /* len + new tokens > cap; that sequence untouched */

/* Layer geometry and switches.  Each switch cites the step it turns on.  */
typedef struct {
  int32_t E;            /* model width */
  int32_t C;            /* compression factor: latent width E / C  [Methodologie 1] */
  int32_t n_q_heads;    /* Hq */
  int32_t n_kv_heads;   /* Hkv; must divide Hq; any group size G = Hq / Hkv
                           (MQA at Hkv = 1, MHA at Hkv = Hq)  [CCGQA; GQA page,
                           "Como funciona GQA"] */
  int32_t conv_width;   /* K in 0..4 taps of the causal sequence conv; 0 = no conv
                           and no channel mix  [Methodologie 2] */
  int32_t qk_mean;      /* QK-mean skip term  [Methodologie 2, QK-Mean]:
                           0 off; 1 "cross": (q~ + k~)/2 of the same position added
                           to q and k (k~ and the mean of the group's q~ for k);
                           2 "self": each head becomes (own pre-conv + conv
                           output) / 2 (the literal reading of the page) */
  int32_t value_shift;  /* value-shift  [Methodologie 3]: 0 off; 1 channels
                           [d/2, d) of every kv head from the previous token;
                           2 whole kv heads: the last floor(Hkv/2) heads from the
                           previous token, the others current */
  int32_t causal;       /* 1 = causal attention mask  [Probleemstelling] */
  double rope_base;     /* RoPE base; 0 = no RoPE  [Methodologie 4] */
  int32_t dtype;        /* ccgqa_dtype: fp32 or bf16; head dim d = E / (C Hq) in
                           {16, 32, 64, 128} for both (bf16 attention runs on the
                           tensor core for d >= 32 and G <= 128, on the CUDA
                           cores otherwise) */
  int32_t channel_conv; /* channel convolution  [Methodologie 2]: 0 = depthwise
                           sequence taps conv_*_seq then one d x d mix per head
                           and position (conv_*_chan [H, d, d], or none); 1 =
                           temporal channel conv with a d x d matrix per tap,
                           y[t] = sum_j W[h, j] z[t - j]: conv_*_chan [H, K, d, d]
                           required, conv_*_seq unused (needs conv_width >= 1) */
} ccgqa_config;

/* Weights (device, cfg->dtype).  [Methodologie 1-2] */
typedef struct {
  /* [N_qkv, E]: output features x input features.  Rows [0, Hq d) give the
     latent queries q~, the next Hkv d rows k~, the last Hkv d rows v~; within
     each block row index = head * d + i.  NULL: the input rows already hold
     q~ | k~ | v~ (width N_qkv) and the projection is skipped. */
  const void* W_qkv;
  /* [Hq d, K]: sequence-conv taps; tap j multiplies the row j steps back. */
  const void* conv_q_seq;
  /* [Hq, d, d]: per-head channel mix y_i = sum_j W[h][i][j] u_j; NULL = none.
     With channel_conv = 1: [Hq, K, d, d], tap j's matrix at [h][j]:
     y[t]_i = sum_j sum_c W[h][j][i][c] z[t-j]_c (conv_q_seq unused). */
  const void* conv_q_chan;
  const void* conv_k_seq;   /* [Hkv d, K] */
  const void* conv_k_chan;  /* [Hkv, d, d]; NULL = none ([Hkv, K, d, d] with channel_conv = 1) */
} ccgqa_weights;

/* Latent KV cache plus the decode state (device buffers, caller-owned).
   [Probleemstelling 2: the cache grows with the sequence; Resultaten 3: it
   shrinks with C.]
   Two layouts of k / v:
    - contiguous (block_table == NULL): k, v are [batch, Hkv, cap, d];
    - paged (block_table != NULL), after "Grouped Query Attention (GQA)",
      section "GQA y tecnicas relacionadas" (PagedAttention: the cache is
      allocated in fixed-size blocks, whatever number of heads fills them):
      k, v are a pool of n_pages pages [n_pages, Hkv, page_size, d], each page
      holding page_size consecutive tokens of one sequence for all Hkv heads.
      Token t of sequence b lives in page block_table[b * (cap / page_size) +
      t / page_size], row t % page_size.  page_size is a power of two from 16
      to 4096 that divides cap; the table has cap / page_size int32 entries per
      sequence, and only the entries of tokens a call reads or writes are
      looked at (the rest may hold anything, e.g. -1 for pages not yet given).
      Pages may be shared between sequences only if no call writes them.  An
      entry outside [0, n_pages) that a kernel needs sets CCGQA_DEVERR_INDEX;
      that access is skipped (writes) or reads zeros (reads), and the
      sequence's output row is then undefined. */
typedef struct {
  void* k;            /* [batch, Hkv, cap, d]  post-RoPE keys (paged: [n_pages, Hkv, page_size, d]) */
  void* v;            /* [batch, Hkv, cap, d]  value-shifted values (paged: as k) */
  int32_t* len;       /* [batch] tokens held (device int32) */
  void* conv_hist_q;  /* [batch, K-1, Hq d]  last K-1 pre-conv q~ rows, oldest first
                         (NULL allowed when K <= 1) */
  void* conv_hist_k;  /* [batch, K-1, Hkv d] */
  void* v_prev;       /* [batch, Hkv d]  last v~ row before the shift (NULL allowed
                         when value_shift == 0) */
  int32_t batch;
  int32_t cap;        /* token capacity per sequence */
  const int32_t* block_table;  /* NULL = contiguous; else [batch, cap / page_size] page ids (device) */
  int32_t page_size;  /* tokens per page (paged only) */
  int32_t n_pages;    /* pages in the pool k / v (paged only; n_pages * Hkv < 2^31) */
} ccgqa_kvcache;

/* Bytes of workspace ccgqa_prefill needs for (batch, seq_len). */
CCGQA_API size_t ccgqa_prefill_workspace_size(const ccgqa_config* cfg, int32_t batch,
                                              int32_t seq_len);

/* Bytes of workspace ccgqa_decode_step needs for a cache of (batch, cap).
   The decode workspace must be zero-filled once before its first use; the
   step leaves it ready for the next one. */
CCGQA_API size_t ccgqa_decode_workspace_size(const ccgqa_config* cfg, int32_t batch,
                                             int32_t cap);

/* Causal prefill of `batch` sequences of `seq_len` tokens from an empty state.
 * x:   [batch, seq_len, E]  (or [batch, seq_len, N_qkv] when w->W_qkv == NULL)
 * out: [batch, seq_len, Hq d]  attention output per query head (no output
 *      projection: the paper's layer ends in the latent space here).
 * cache: nullable.  When given, rows [0, seq_len) of cache->k / cache->v are
 *      overwritten, len[b] = seq_len, and the conv histories and v_prev are set
 *      so that ccgqa_decode_step continues the sequences.  Needs
 *      seq_len <= cache->cap and cache->batch == batch (else CCGQA_ERR_CAPACITY
 *      / CCGQA_ERR_INVALID_ARG).  A paged cache is filled after the attention
 *      (which reads k / v from the workspace) by one page-scatter kernel.
 * workspace: >= ccgqa_prefill_workspace_size bytes, 256-byte aligned.
 * Steps: projection (tcgen05 GEMM for bf16), fused conv + channel mix +
 * QK-mean + RoPE + value-shift, flash attention (tcgen05/TMEM/TMA for bf16).
 * For bf16 at d = 32 with the depthwise conv (conv_width 1-4, both channel
 * mixes given, G <= 6) the projection and the steps after it run as one
 * kernel whose projected rows stay in shared memory; its results equal the
 * separate kernels' bit for bit (ccgqa_set_fused_projection turns it off). */
CCGQA_API ccgqa_status ccgqa_prefill(const ccgqa_config* cfg, const ccgqa_weights* w,
                                     const void* x, int32_t batch, int32_t seq_len,
                                     void* out, const ccgqa_kvcache* cache,
                                     void* workspace, size_t workspace_bytes,
                                     int32_t* dev_err, void* stream);

/* One new token per sequence against the latent KV cache: equals row len[b]
 * of a prefill over all tokens so far.
 * x_t: [batch, E] (or [batch, N_qkv] when w->W_qkv == NULL);
 * out: [batch, Hq d].  Appends the new k/v row at len[b], updates the conv
 * histories and v_prev, then len[b] += 1.  A sequence with len[b] >= cap sets
 * CCGQA_DEVERR_CAPACITY and is left unchanged (its out row is zero).
 * workspace: >= ccgqa_decode_workspace_size(cfg, cache->batch, cache->cap),
 * zero-filled before first use.  Steps that overlap on the GPU and share one
 * workspace race; give concurrent streams their own workspace. */
CCGQA_API ccgqa_status ccgqa_decode_step(const ccgqa_config* cfg, const ccgqa_weights* w,
                                         const void* x_t, const ccgqa_kvcache* cache,
                                         void* out, void* workspace,
                                         size_t workspace_bytes, int32_t* dev_err,
                                         void* stream);

/* ccgqa_decode_step without a caller-provided workspace.  The paper has no
 * counterpart: this is a deployment convenience.  Some callers cannot
 * allocate device memory -- for example a serving runtime whose memory plan is
 * fixed up front and owned entirely by its own allocator, or a host that only
 * lends this library existing buffers and has no way to hand it a new one.
 * This entry point takes the same inputs and outputs as ccgqa_decode_step
 * (no workspace arguments) and uses instead a scratch array compiled into the
 * library: ccgqa_decode_noalloc_max_bytes() bytes (16 MiB) of device global
 * memory, held by each GPU from the moment the library's module is loaded on
 * it until the process exits.
 *  - When the module loads: CUDA loads modules lazily by default (since
 *    CUDA 12.2, CUDA_MODULE_LOADING=LAZY), so the array is placed on a device
 *    by the first call of this entry point there, not when the library is
 *    opened.  That first call therefore takes 16 MiB from the device; with an
 *    eager module-loading setting the array is placed at context creation.
 *    Callers with a fixed memory plan should make one warm-up call on each
 *    device at initialisation, before their plan is fixed and before any
 *    stream capture; later calls take no device memory.
 *  - Returns CCGQA_ERR_WORKSPACE when the decode needs more scratch than that
 *    (see ccgqa_decode_workspace_size); it never allocates, frees or calls an
 *    allocating library routine.
 *  - The first call on each device also looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current).
 *  - All calls share the one array and it keeps the last call's contents: the
 *    call clears the parts that must start at zero itself, but calls whose work
 *    overlaps on the GPU (other streams, other host threads) race on it --
 *    order them, or use ccgqa_decode_step with separate workspaces. */
CCGQA_API ccgqa_status ccgqa_decode_step_noalloc(const ccgqa_config* cfg, const ccgqa_weights* w,
                                                 const void* x_t, const ccgqa_kvcache* cache,
                                                 void* out, int32_t* dev_err, void* stream);

/* Scratch bytes available to ccgqa_decode_step_noalloc. */
CCGQA_API size_t ccgqa_decode_noalloc_max_bytes(void);

/* Append n_new rows per sequence: cache->k[b, g, len[b] + i, :] = k_new[b, i, g, :]
 * (same for v; in a paged cache, token len[b] + i of sequence b at its page
 * and row), then len[b] += n_new.  Bit-exact copy.
 * k_new, v_new: [batch, n_new, Hkv, d].  n_new > cap returns CCGQA_ERR_CAPACITY
 * on the host; a sequence whose len[b] + n_new > cap is skipped on the device
 * and sets CCGQA_DEVERR_CAPACITY.  Conv histories and v_prev are not touched. */
CCGQA_API ccgqa_status ccgqa_kvcache_append(const ccgqa_config* cfg, const ccgqa_kvcache* cache,
                                            const void* k_new, const void* v_new,
                                            int32_t n_new, int32_t* dev_err, void* stream);

/* Gradient buffers of the layer's weights for ccgqa_prefill_backward: fp32,
 * device, caller-owned, each with the shape of its weight (conv_*_chan of the
 * temporal channel conv included).  Any entry may be NULL (that gradient is
 * not computed); the call zero-fills the others and then writes them. */
typedef struct {
  float* W_qkv;         /* [N_qkv, E] */
  float* conv_q_seq;    /* [Hq d, K] (depthwise taps) */
  float* conv_q_chan;   /* [Hq, d, d], or [Hq, K, d, d] with channel_conv = 1 */
  float* conv_k_seq;    /* [Hkv d, K] */
  float* conv_k_chan;   /* [Hkv, d, d], or [Hkv, K, d, d] with channel_conv = 1 */
} ccgqa_weight_grads;

/* Workspace bytes of ccgqa_prefill_backward for `batch` sequences of
 * `seq_len` tokens (0 on an invalid configuration). */
CCGQA_API size_t ccgqa_prefill_backward_workspace_size(const ccgqa_config* cfg, int32_t batch,
                                                       int32_t seq_len);

/* Backward pass of ccgqa_prefill (from an empty state, no cache): given the
 * gradient dout of the prefill's output, the gradient of the input and of the
 * weights.  The CCA page ("Compressed Convolutional Attention", Resultaten 2)
 * trains the layer and reports its backward pass; its steps are the
 * transposes of the forward steps in reverse order: attention (dQ, dK, dV,
 * with a kv head's gradients summed over its G query heads), value-shift,
 * RoPE, QK-mean, channel mix or temporal channel conv, sequence conv,
 * projection.
 *  - x:    [batch, seq_len, E] (or the packed q~|k~|v~ rows when W_qkv is NULL),
 *          the same input the forward was given;
 *  - dout: [batch, seq_len, Hq*d], gradient of the prefill output;
 *  - dx:   [batch, seq_len, E] (or [batch, seq_len, N_qkv]) written, cfg->dtype;
 *  - dw:   weight gradients (fp32), nullable.
 * x, dout and dx in cfg->dtype, 16-byte aligned, device, caller-owned; dx must
 * not overlap x or dout.  The forward values the backward needs (projection
 * output, q, k, v) are recomputed into the workspace (>= the size above,
 * 256-byte aligned).  Every gradient is accumulated in fp32 on the CUDA cores;
 * the bf16 path uses the same bf16-rounded q, k and v the forward uses.
 * Returns the same host-side statuses as ccgqa_prefill (INVALID_ARG,
 * UNSUPPORTED, WORKSPACE), CCGQA_ERR_CUDA on a launch failure, else CCGQA_OK
 * (asynchronous on `stream`).  The weight gradients are sums over positions
 * with atomic adds for the sequence-conv taps, so those bits may differ
 * between runs; everything else is deterministic. */
CCGQA_API ccgqa_status ccgqa_prefill_backward(const ccgqa_config* cfg, const ccgqa_weights* w,
                                              const void* x, int32_t batch, int32_t seq_len,
                                              const void* dout, void* dx,
                                              const ccgqa_weight_grads* dw, void* workspace,
                                              size_t workspace_bytes, int32_t* dev_err,
                                              void* stream);

/* Output up-projection: the latent attention output mapped back to the model
 * width E.  The CCA page ("Compressed Convolutional Attention", Methodologie
 * item 1) runs the whole attention inside the latent space and leaves the way
 * back to width E unstated; the reading here is one bias-free linear map:
 *   y[m, e] = sum_j o[m, j] * W_o[e, j],   m < M, j < Hq*d, e < E.
 *  - o:   [M, Hq*d] device, e.g. ccgqa_prefill's out viewed as [batch*seq_len,
 *         Hq*d] or ccgqa_decode_step's out ([batch, Hq*d]);
 *  - W_o: [E, Hq*d] device, output-feature major (like W_qkv);
 *  - y:   [M, E] device, written; must not overlap o or W_o.
 * All three in cfg->dtype and 16-byte aligned, caller-owned.  bf16: tcgen05
 * GEMM with fp32 accumulation, y rounded to bf16 once; f32: fp32 GEMM on the
 * CUDA cores.  Only E, C, n_q_heads and dtype of cfg are used (validated as
 * for every call).  Returns CCGQA_ERR_INVALID_ARG for M <= 0, a NULL or
 * misaligned pointer, or another stream while this thread records a graph;
 * CCGQA_ERR_UNSUPPORTED for M > 2^30 or (bf16) Hq*d not a multiple of 8;
 * CCGQA_ERR_CUDA on a launch failure; else CCGQA_OK (asynchronous on
 * `stream`; a bounded wait that runs out sets CCGQA_DEVERR_TIMEOUT in
 * *dev_err, nullable). */
CCGQA_API ccgqa_status ccgqa_output_projection(const ccgqa_config* cfg, const void* W_o,
                                               const void* o, int64_t M, void* y,
                                               int32_t* dev_err, void* stream);

/* Static description of a status code. */
CCGQA_API const char* ccgqa_status_string(ccgqa_status s);

/* Name and description of the last CUDA error an entry point met on the
 * calling thread (after it returned CCGQA_ERR_CUDA); "no error" otherwise. */
CCGQA_API const char* ccgqa_last_error_string(void);

/* Number of kernels this library has launched in this process. */
CCGQA_API uint64_t ccgqa_launch_count(void);

/* Optional timing hook for the calling host thread.  `events` points to n >= 4
 * cudaEvent_t handles created by the caller; while set, ccgqa_prefill records
 * events[0] before its first kernel, events[1] after the projection, events[2]
 * after the pre-attention kernel and events[3] after attention, and
 * ccgqa_decode_step records the same four points around its projection,
 * pre-step and attention kernels -- all on the call's stream.  NULL or n < 4
 * turns it off.  Only the pointer is kept; the caller keeps the events alive. */
CCGQA_API void ccgqa_set_phase_events(void* const* events, int32_t n);

/* Process-wide switch (default 1 = on).  When on, ccgqa_prefill runs the
 * latent projection and the pre-attention steps as ONE kernel where that
 * kernel applies: bf16, d = 32, a projection weight, conv width 1..4 with
 * depthwise taps and both channel-mix weights, G <= 6, 16-byte aligned x, W
 * and conv weights ("Compressed Convolutional Attention", Methodologie: the
 * projected q~ | k~ | v~ never reach HBM).  Its phase events [1] and [2] then
 * both fall after that kernel.  0 runs the projection GEMM and the
 * pre-attention kernel separately (the same results, bit for bit: the fused
 * kernel rounds the projection to bf16 as the GEMM does and repeats the later
 * steps' arithmetic).  For measurement and testing. */
CCGQA_API void ccgqa_set_fused_projection(int32_t enable);

/* Self-test of the device-side failure reporting (no counterpart in the
 * papers; it exercises the bounded wait every kernel of this library uses).
 * Launches one small kernel on `stream` whose threads wait on an mbarrier that
 * nothing ever arrives on; each wait gives up after about `limit_cycles` SM
 * clock cycles (1 <= limit_cycles <= 2e9), and the kernel then ORs
 * CCGQA_DEVERR_TIMEOUT into *dev_err (device, nullable) and returns, leaving
 * the CUDA context usable.  Returns CCGQA_ERR_INVALID_ARG for a limit out of
 * range, CCGQA_ERR_CUDA if the launch fails, else CCGQA_OK (asynchronous: read
 * *dev_err after synchronising the stream). */
CCGQA_API ccgqa_status ccgqa_selftest_wait_timeout(int64_t limit_cycles, int32_t* dev_err,
                                                   void* stream);

/* CUDA graphs of library calls (no counterpart in the papers: a launch-cost
 * device for fixed-shape serving loops, where one graph launch replaces the
 * per-kernel launches of a prefill and a decode step).
 *
 * ccgqa_graph_begin starts recording on `stream` (a created stream: NULL, the
 * legacy and the per-thread default streams return CCGQA_ERR_INVALID_ARG) in
 * thread-local capture mode.  Until ccgqa_graph_end, the calling thread's
 * ccgqa_prefill / ccgqa_decode_step / ccgqa_decode_step_noalloc /
 * ccgqa_kvcache_append / ccgqa_selftest_wait_timeout calls validate their
 * arguments as usual but only RECORD their kernels, which do not run; a call
 * that names another stream returns CCGQA_ERR_INVALID_ARG, and phase events
 * (ccgqa_set_phase_events) are not recorded.  Other work the caller puts on the
 * stream meanwhile (copies, its own kernels) is recorded too.  A second begin
 * on the same thread before end returns CCGQA_ERR_INVALID_ARG.
 *
 * ccgqa_graph_end(stream, &graph) stops recording and instantiates the graph;
 * *graph receives a handle the caller owns (free it with ccgqa_graph_destroy).
 * Errors: CCGQA_ERR_INVALID_ARG if this thread is not recording on `stream` or
 * graph is NULL; CCGQA_ERR_CUDA if the capture was invalidated or
 * instantiation failed (*graph = NULL, recording has stopped either way).
 *
 * ccgqa_graph_launch(graph, stream) runs the recorded work once on `stream`
 * (any stream of the graph's device), with every pointer and size exactly as
 * recorded: to run on new inputs, write them into the recorded buffers
 * first.  The device error word and the cache are updated as by the recorded
 * calls.  Launch order on a stream is the only ordering; two launches of one
 * graph must not overlap in time.  Each launch adds the graph's kernel count to
 * ccgqa_launch_count (recording adds nothing).
 *
 * ccgqa_graph_kernel_count: library kernels one launch runs (-1 for NULL).
 * ccgqa_graph_destroy: frees the graph (NULL is a no-op); the caller makes sure
 * no launch of it is still running. */
typedef struct ccgqa_graph ccgqa_graph;
CCGQA_API ccgqa_status ccgqa_graph_begin(void* stream);
CCGQA_API ccgqa_status ccgqa_graph_end(void* stream, ccgqa_graph** graph);
CCGQA_API ccgqa_status ccgqa_graph_launch(const ccgqa_graph* graph, void* stream);
CCGQA_API int64_t ccgqa_graph_kernel_count(const ccgqa_graph* graph);
CCGQA_API ccgqa_status ccgqa_graph_destroy(ccgqa_graph* graph);

#ifdef __cplusplus
}
#endif

#endif /* CCGQA_H */
