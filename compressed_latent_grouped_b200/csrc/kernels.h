// Internal launcher declarations shared by the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace ccgqa {

using bf16 = __nv_bfloat16;

// ----------------------------------------------------------------- tensor maps
// Encode a tiled TMA descriptor through the driver entry point (no libcuda link).
// dims / box are innermost-first; strides_bytes has rank-1 entries (dims 1..).
bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                       const uint64_t* dims, const uint64_t* strides_bytes,
                       const uint32_t* box, CUtensorMapSwizzle swizzle);

// ----------------------------------------------------------------- projection
// C[M, N] = A[M, K] * W[N, K]^T, bf16 in / fp32 accumulate / bf16 out (tcgen05).
// A, W, C 16-byte aligned, K and N multiples of 8 (TMA row pitches; N % 8 != 0
// returns cudaErrorInvalidValue).
cudaError_t launch_proj_gemm_bf16(const bf16* A, const bf16* W, bf16* C, int M, int N, int K,
                                  int32_t* dev_err, cudaStream_t stream);
// The same tensor-core GEMM with an fp32 output (N % 4 == 0).
cudaError_t launch_gemm_bf16_f32out(const bf16* A, const bf16* W, float* C, int M, int N, int K,
                                    int32_t* dev_err, cudaStream_t stream);
// Same contraction in fp32 on the CUDA cores.
cudaError_t launch_proj_gemm_f32(const float* A, const float* W, float* C, int M, int N, int K,
                                 cudaStream_t stream);

// ----------------------------------------------------------------- pre-attention
template <typename T>
struct PreAttnArgs {
  const T* src;          // [B*S, src_ld] rows: q~ | k~ | v~ columns
  int64_t src_ld;
  int B, S, Hq, Hkv, d, G, K;   // K = conv width, 0 = no conv / channel mix
  int qk_mean;           // 0 off, 1 cross (q~ + k~) / 2 added, 2 self (y + own pre) / 2
  int value_shift;       // 0 off, 1 upper half-channels, 2 last floor(Hkv / 2) kv heads
  int channel_conv;      // 1: per-tap d x d matrices (wq_chan [Hq, K, d, d]), no depthwise taps
  int rope_on;
  double rope_log2_base;
  // theta_i / (2 pi) as a 0.64 fixed-point fraction of a turn, i < d/2: the
  // product t * rope_frac[i] modulo 2^64 is the angle t * theta_i reduced
  // modulo one turn, exactly (used by the tensor-core pre-attention kernel)
  uint64_t rope_frac[64];
  const T *wq_seq, *wq_chan, *wk_seq, *wk_chan;  // chan may be null
  T* q_out;              // [B, S, Hq, d]
  T* k_out;              // [B, Hkv, kv_cap, d]
  T* v_out;
  int64_t kv_cap;
  T* hist_q;             // nullable decode state
  T* hist_k;
  T* v_prev;
  int32_t* len;
  int32_t* dev_err;
};
template <typename T>
cudaError_t launch_pre_attn(const PreAttnArgs<T>& a, cudaStream_t stream);
// Whether the CUDA-core pre-attention kernel's smallest staging layout (8
// positions per CTA) fits in shared memory for this group size and head dim.
bool pre_attn_fits(int K, int G, int d, int es, bool has_mix);
// bf16, d in {32, 64}, conv 1..4 taps with both channel-mix weights, 16-byte
// aligned inputs and weights, the layout within 227 KB of shared memory: the mix
// on tcgen05, staging by TMA (launch_pre_attn dispatches there when this holds).
bool pre_attn_tc_supported(const PreAttnArgs<bf16>& a);
cudaError_t launch_pre_attn_tc(const PreAttnArgs<bf16>& a, cudaStream_t stream);
// The projection fused with the pre-attention (bf16, d = 32, G <= 6, conv 1..4
// taps with both channel-mix weights): x [B, S, E] and W [N, E] in, a.src unused.
bool proj_pre_tc_supported(const PreAttnArgs<bf16>& a, const bf16* x, const bf16* W, int E);
cudaError_t launch_proj_pre_tc(const bf16* x, const bf16* W, int E, const PreAttnArgs<bf16>& a,
                               cudaStream_t stream);

// ----------------------------------------------------------------- attention
struct AttnArgs {
  const void* q;         // [B, S, Hq, d]
  const void* k;         // [B, Hkv, kv_cap, d]
  const void* v;
  void* out;             // [B, S, Hq, d]
  int B, S, Hq, Hkv, d, G;
  int64_t kv_cap;
  int causal;
  int32_t* dev_err;
  // optional (tensor-core kernel only): each stored row's log-sum-exp in base
  // 2 of the scaled scores, negated, -log2(sum_s 2^(log2(e) q.k_s / sqrt(d))),
  // at lse[(b Hkv + g) lse_ld + t G + head in group]
  float* lse = nullptr;
  int64_t lse_ld = 0;
};
// bf16, d in {32, 64, 128}, any G <= 128 (a tile holds floor(128 / G)
// positions of the group's G heads): tcgen05/TMEM/TMA flash attention.
cudaError_t launch_attn_prefill_tc(const AttnArgs& a, cudaStream_t stream);

// Attention backward on the tensor core (bf16, d in {32, 64, 128}, G a power
// of two up to 64).  lse / dsum: [B Hkv, ld] packed per (sequence, kv group),
// row t G + head in group, ld a multiple of 64 of at least S G, both negated:
// lse from the forward kernel, dsum written here (-D, D = rowsum(dO o)).
struct AttnBwdTcArgs {
  const void *q, *k, *v, *o, *dout;   // q, o, dout [B, S, Hq, d]; k, v [B, Hkv, S, d]
  const float* lse;
  float* dsum;
  int64_t ld;
  float *dq, *dk, *dv;                // fp32, like q, k, v
  int B, S, Hq, Hkv, d, G, causal;
  int32_t* dev_err;
};
bool attn_bwd_tc_supported(int d, int G);
cudaError_t launch_attn_bwd_tc(const AttnBwdTcArgs& a, cudaStream_t stream);
// CUDA-core flash attention (the fp32 path; bf16 where the tensor-core kernel
// does not apply: d = 16 or G > 128).
template <typename T>
cudaError_t launch_attn_prefill_simt(const AttnArgs& a, cudaStream_t stream);

// ----------------------------------------------------------------- cache + decode
// Where token t of (sequence b, kv head g) sits in the cache's k / v buffers.
// Contiguous (table == null): [B, Hkv, cap, d].  Paged: a pool [n_pages, Hkv,
// 2^shift, d] and a block table [B, per_seq] naming the page of every
// 2^shift consecutive tokens of a sequence.
struct PageMap {
  const int32_t* table;
  int per_seq;           // table entries per sequence (cap >> shift)
  int shift;             // log2(page size)
  int n_pages;
};
// Row (in units of d elements) of token t of (b, g), or -1 when the page id the
// table gives is outside the pool.
__device__ __forceinline__ int64_t kv_row(const PageMap& pm, int b, int g, int Hkv, int64_t cap,
                                          int64_t t) {
  if (pm.table == nullptr) return (static_cast<int64_t>(b) * Hkv + g) * cap + t;
  const int pg = __ldg(pm.table + static_cast<int64_t>(b) * pm.per_seq + (t >> pm.shift));
  if (pg < 0 || pg >= pm.n_pages) return -1;
  return ((static_cast<int64_t>(pg) * Hkv + g) << pm.shift) + (t & ((int64_t{1} << pm.shift) - 1));
}

// Append n_new rows per sequence at len[b] (then len[b] += n_new): k_new, v_new
// [B, n_new, Hkv, d].
template <typename T>
cudaError_t launch_kv_append(T* cache_k, T* cache_v, const PageMap& pm, int32_t* len,
                             const T* k_new, const T* v_new, int B, int Hkv, int d, int64_t cap,
                             int n_new, int32_t* dev_err, cudaStream_t stream);
// Copy rows [0, S) of k_src, v_src [B, Hkv, S, d] into a paged cache (len untouched).
template <typename T>
cudaError_t launch_kv_scatter(T* cache_k, T* cache_v, const PageMap& pm, const T* k_src,
                              const T* v_src, int B, int Hkv, int d, int64_t cap, int S,
                              int32_t* dev_err, cudaStream_t stream);

template <typename T>
struct DecodeArgs {
  const T* x_t;          // [B, E] or packed [B, N] when W is null
  const T* W;            // [N, E] or null
  int B, E, N, Hq, Hkv, d, G, K;
  int qk_mean, value_shift, causal, rope_on;   // modes as in PreAttnArgs
  int channel_conv;
  double rope_log2_base;
  uint64_t rope_frac[64];  // theta_i / (2 pi) in 0.64 fixed point, i < d/2 (see PreAttnArgs)
  const T *wq_seq, *wq_chan, *wk_seq, *wk_chan;
  T* cache_k;            // [B, Hkv, cap, d], or a page pool (see PageMap)
  T* cache_v;
  PageMap pages;
  int32_t* len;
  int64_t cap;
  T* hist_q;             // [B, K-1, Hq d]
  T* hist_k;             // [B, K-1, Hkv d]
  T* v_prev;             // [B, Hkv d]
  T* out;                // [B, Hq d]
  // workspace pieces
  float* proj_part;      // [e_splits, B, N]
  int e_splits;
  float* q_ws;           // [B, Hq, d]
  float* part_o;         // [B, Hkv, splits, G, d]
  float* part_ml;        // [B, Hkv, splits, G, 2]
  int32_t* tickets;      // [B*Hkv + B], zero before the first step, left zero after
  int splits;
  int chunk;             // keys per split
  int32_t* dev_err;
  void* const* phase_events;  // optional: 4 cudaEvent_t recorded between the kernels
};
template <typename T>
cudaError_t launch_decode_step(const DecodeArgs<T>& a, cudaStream_t stream);
// bf16 decode attention on the tensor core (d in {32, 64, 128}, G <= 16).
cudaError_t launch_decode_attn_tc(const DecodeArgs<bf16>& a, cudaStream_t stream);

// Whether the one-token pre-step's shared memory (without staged mix weights)
// fits for this group size and head dim.
bool decode_pre_fits(int G, int d, int K, int es);

// ----------------------------------------------------------------- backward
// Backward pass of a prefill (ccgqa_prefill_backward).  Forward values z, q,
// k, v were recomputed into the workspace; every gradient buffer is fp32.
template <typename T>
struct BwdArgs {
  int B, S, E, N, Hq, Hkv, d, G, K;
  int qk_mean, value_shift, causal, rope_on, channel_conv;
  uint64_t rope_frac[64];      // as in PreAttnArgs
  const T* x;                  // [B S, E] (or the packed rows when W is null)
  const T* W;                  // [N, E] or null
  const T *wq_seq, *wq_chan, *wk_seq, *wk_chan;
  const T* z;                  // [B S, N] q~ | k~ | v~ (the projection output, or x)
  const T *q, *k, *v;          // [B, S, Hq, d], [B, Hkv, S, d] x 2
  const T* dout;               // [B, S, Hq, d]
  float *dq, *dk, *dv;         // like q, k, v
  float *lse, *dsum;           // [B, Hq, S]: log-sum-exp and rowsum(dO * O)
                               // (tensor-core path: [B Hkv, lse_ld] packed rows)
  int64_t lse_ld;
  T* o;                        // [B, S, Hq, d] forward output (tensor-core path)
  int32_t* dev_err;
  // bf16 with a projection: the gradient GEMMs on the tensor core read
  // dz_b = bf16(dz) [B S, N], W^T [E, N], and dz^T [N, ldr], x^T [E, ldr]
  // (ldr = B S rounded up to a multiple of 8, zero past B S); null otherwise
  T *dz_b, *WT, *dzT, *xT;
  int64_t ldr;
  float *dy, *dzm, *du, *u;    // [B S, (Hq + Hkv) d]
  float* dz;                   // [B S, N]
  T* dx;                       // [B S, E] (or [B S, N] for packed input)
  float *g_W, *g_q_seq, *g_q_chan, *g_k_seq, *g_k_chan;   // nullable, zeroed first
};
template <typename T>
cudaError_t launch_backward(const BwdArgs<T>& a, cudaStream_t stream);

// Split plan for the decode step, shared by the workspace-size query and the launch.
void decode_plan(int B, int Hkv, int E, int N, int64_t cap, bool has_proj, int es,
                 int* e_splits, int* splits, int* chunk);

}  // namespace ccgqa
