// Grouped-query causal attention on the CUDA cores, for the fp32 path (fp32
// operands must not be rounded to a tensor-core input type).
// ("Compressed Convolutional Attention", CCGQA; "Grouped Query Attention
// (GQA)", "Cómo funciona GQA".)
//
// One CTA = 32 query positions of one query head; 4 threads per position, each
// holding d/4 interleaved dims of q and of the running output.  K/V tiles of 64
// keys are staged in shared memory; scores are reduced over the 4 threads with
// shuffles and folded into an online softmax per key.
#include "kernels.h"

namespace ccgqa {
namespace {

constexpr int kRows = 32, kSub = 4;

template <typename T, int D>
__global__ void __launch_bounds__(kRows * kSub)
    attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     T* __restrict__ out, int S, int Hq, int Hkv, int G, int64_t cap,
                     int causal) {
  constexpr int DS = D / kSub;
  constexpr int kKeys = D <= 64 ? 64 : 32;  // keeps the K/V stage under 48 KB
  __shared__ float Ks[kKeys][D + 1];
  __shared__ float Vs[kKeys][D + 1];
  const int b = blockIdx.z, h = blockIdx.y, g = h / G;
  const int row = threadIdx.x / kSub, sub = threadIdx.x % kSub;
  const int t = blockIdx.x * kRows + row;
  const bool valid = t < S;
  const T* kb = k + (static_cast<int64_t>(b) * Hkv + g) * cap * D;
  const T* vb = v + (static_cast<int64_t>(b) * Hkv + g) * cap * D;
  float qr[DS], o[DS];
  const float scale = rsqrtf(static_cast<float>(D));
#pragma unroll
  for (int i = 0; i < DS; ++i) {
    qr[i] = valid ? to_f32(q[((static_cast<int64_t>(b) * S + t) * Hq + h) * D + sub + kSub * i]) *
                        scale
                  : 0.f;
    o[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int t_hi = min(blockIdx.x * kRows + kRows - 1, S - 1);
  const int n_keys = causal ? t_hi + 1 : S;
  for (int s0 = 0; s0 < n_keys; s0 += kKeys) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kKeys * D; idx += kRows * kSub) {
      const int r = idx / D, c = idx % D;
      const int s = s0 + r;
      Ks[r][c] = s < S ? to_f32(kb[static_cast<int64_t>(s) * D + c]) : 0.f;
      Vs[r][c] = s < S ? to_f32(vb[static_cast<int64_t>(s) * D + c]) : 0.f;
    }
    __syncthreads();
    const int lim = min(kKeys, n_keys - s0);
    for (int c = 0; c < lim; ++c) {
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < DS; ++i) part = fmaf(qr[i], Ks[c][sub + kSub * i], part);
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      const int s = s0 + c;
      if (!valid || (causal && s > t) || s >= S) continue;
      const float m_new = fmaxf(m, part);
      const float corr = expf(m - m_new);
      const float p = expf(part - m_new);
      l = l * corr + p;
#pragma unroll
      for (int i = 0; i < DS; ++i) o[i] = fmaf(p, Vs[c][sub + kSub * i], o[i] * corr);
      m = m_new;
    }
  }
  if (valid) {
    const float inv = 1.f / l;
#pragma unroll
    for (int i = 0; i < DS; ++i)
      out[((static_cast<int64_t>(b) * S + t) * Hq + h) * D + sub + kSub * i] =
          from_f32<T>(o[i] * inv);
  }
}

template <typename T, int D>
cudaError_t launch_simt_d(const AttnArgs& a, cudaStream_t stream) {
  dim3 grid((a.S + kRows - 1) / kRows, a.Hq, a.B);
  attn_simt_kernel<T, D><<<grid, kRows * kSub, 0, stream>>>(
      static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v),
      static_cast<T*>(a.out), a.S, a.Hq, a.Hkv, a.G, a.kv_cap, a.causal);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

template <typename T>
cudaError_t launch_attn_prefill_simt(const AttnArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 16: return launch_simt_d<T, 16>(a, stream);
    case 32: return launch_simt_d<T, 32>(a, stream);
    case 64: return launch_simt_d<T, 64>(a, stream);
    case 128: return launch_simt_d<T, 128>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

template cudaError_t launch_attn_prefill_simt<float>(const AttnArgs&, cudaStream_t);
template cudaError_t launch_attn_prefill_simt<bf16>(const AttnArgs&, cudaStream_t);

}  // namespace ccgqa
