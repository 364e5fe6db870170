// Backward pass of the CCGQA layer on the CUDA cores ("Compressed Convolutional
// Attention", Resultaten 2: the layer is trained, so its backward pass runs
// on the same hardware; the steps are the transposes of the forward steps in
// reverse order).  Every gradient is accumulated in fp32; the forward values
// the backward needs are recomputed by the forward kernels (projection,
// pre-attention) into the workspace.
//
//   attention    dQ pass (query-major: recomputes O and the log-sum-exp, then
//                D = rowsum(dO * O) and dQ) and dK/dV pass (key-major, summing
//                over the G query heads of the group, no atomics)
//   rows         RoPE transpose, QK-mean transpose, value-shift transpose
//   mix / conv   transpose of the per-head channel mix, of the depthwise
//                sequence conv (anti-causal), or of the temporal channel conv
//   weights      tap gradients by a segmented reduction, channel-matrix and
//                projection gradients and dx by one strided GEMM
#include "kernels.h"

namespace ccgqa {
namespace {

constexpr int kRows = 32, kSub = 4;

// ----------------------------------------------------------------- attention
// dQ pass: one CTA = 32 query positions of one query head, 4 threads per
// position with d/4 interleaved dims of q, dO, O and dQ.  Pass 1 is the
// forward's online softmax (O and the row's log-sum-exp); pass 2 rereads the
// keys: p = exp(s - lse), dp = dO . v, ds = p (dp - D), dQ += ds k / sqrt(d).
template <typename T, int D>
__global__ void __launch_bounds__(kRows * kSub)
    attn_bwd_dq_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                       const T* __restrict__ dout, float* __restrict__ dq,
                       float* __restrict__ lse_out, float* __restrict__ dsum_out, int S, int Hq,
                       int Hkv, int G, int causal) {
  constexpr int DS = D / kSub;
  constexpr int kKeys = D <= 64 ? 64 : 32;
  __shared__ float Ks[kKeys][D + 1];
  __shared__ float Vs[kKeys][D + 1];
  const int b = blockIdx.z, h = blockIdx.y, g = h / G;
  const int row = threadIdx.x / kSub, sub = threadIdx.x % kSub;
  const int t = blockIdx.x * kRows + row;
  const bool valid = t < S;
  const T* kb = k + (static_cast<int64_t>(b) * Hkv + g) * S * D;
  const T* vb = v + (static_cast<int64_t>(b) * Hkv + g) * S * D;
  const int64_t qrow = ((static_cast<int64_t>(b) * S + t) * Hq + h) * D;
  const float scale = rsqrtf(static_cast<float>(D));
  float qr[DS], dor[DS], o[DS], dqa[DS];
#pragma unroll
  for (int i = 0; i < DS; ++i) {
    qr[i] = valid ? to_f32(q[qrow + sub + kSub * i]) * scale : 0.f;
    dor[i] = valid ? to_f32(dout[qrow + sub + kSub * i]) : 0.f;
    o[i] = 0.f;
    dqa[i] = 0.f;
  }
  const int t_hi = min(blockIdx.x * kRows + kRows - 1, S - 1);
  const int n_keys = causal ? t_hi + 1 : S;
  auto stage = [&](int s0) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kKeys * D; idx += kRows * kSub) {
      const int r = idx / D, c = idx % D;
      const int s = s0 + r;
      Ks[r][c] = s < S ? to_f32(kb[static_cast<int64_t>(s) * D + c]) : 0.f;
      Vs[r][c] = s < S ? to_f32(vb[static_cast<int64_t>(s) * D + c]) : 0.f;
    }
    __syncthreads();
  };
  auto dot4 = [&](const float (&a)[DS], const float* row_s) {
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < DS; ++i) part = fmaf(a[i], row_s[sub + kSub * i], part);
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    part += __shfl_xor_sync(0xffffffffu, part, 2);
    return part;
  };
  // pass 1: online softmax -> O, lse
  float m = -INFINITY, l = 0.f;
  for (int s0 = 0; s0 < n_keys; s0 += kKeys) {
    stage(s0);
    const int lim = min(kKeys, n_keys - s0);
    for (int c = 0; c < lim; ++c) {
      const float sc = dot4(qr, Ks[c]);
      const int s = s0 + c;
      if (!valid || (causal && s > t) || s >= S) continue;
      const float m_new = fmaxf(m, sc);
      const float corr = expf(m - m_new);
      const float p = expf(sc - m_new);
      l = l * corr + p;
#pragma unroll
      for (int i = 0; i < DS; ++i) o[i] = fmaf(p, Vs[c][sub + kSub * i], o[i] * corr);
      m = m_new;
    }
  }
  const float lse = m + logf(l);
  float dsum = 0.f;
#pragma unroll
  for (int i = 0; i < DS; ++i) dsum = fmaf(dor[i], o[i], dsum);
  dsum += __shfl_xor_sync(0xffffffffu, dsum, 1);
  dsum += __shfl_xor_sync(0xffffffffu, dsum, 2);
  dsum /= l;
  // pass 2: dQ
  for (int s0 = 0; s0 < n_keys; s0 += kKeys) {
    stage(s0);
    const int lim = min(kKeys, n_keys - s0);
    for (int c = 0; c < lim; ++c) {
      const float sc = dot4(qr, Ks[c]);
      const float dp = dot4(dor, Vs[c]);
      const int s = s0 + c;
      if (!valid || (causal && s > t) || s >= S) continue;
      const float ds = expf(sc - lse) * (dp - dsum);
#pragma unroll
      for (int i = 0; i < DS; ++i) dqa[i] = fmaf(ds, Ks[c][sub + kSub * i], dqa[i]);
    }
  }
  if (valid) {
#pragma unroll
    for (int i = 0; i < DS; ++i) dq[qrow + sub + kSub * i] = dqa[i] * scale;
    if (sub == 0) {
      const int64_t lr = (static_cast<int64_t>(b) * Hq + h) * S + t;
      lse_out[lr] = lse;
      dsum_out[lr] = dsum;
    }
  }
}

// dK/dV pass: one CTA = 32 keys of one kv group, 4 threads per key with d/4
// interleaved dims of k, v, dK and dV.  Query rows that see the keys (all
// later positions when causal) are staged 32 positions at a time for each of
// the G heads of the group: p = exp(s - lse), dV += p dO,
// ds = p (dO . v - D), dK += ds q / sqrt(d).
template <typename T, int D>
__global__ void __launch_bounds__(kRows * kSub)
    attn_bwd_dkdv_kernel(const T* __restrict__ q, const T* __restrict__ k,
                         const T* __restrict__ v, const T* __restrict__ dout,
                         const float* __restrict__ lse_in, const float* __restrict__ dsum_in,
                         float* __restrict__ dk, float* __restrict__ dv, int S, int Hq, int Hkv,
                         int G, int causal) {
  constexpr int DS = D / kSub;
  __shared__ float Qs[kRows][D + 1];
  __shared__ float Os[kRows][D + 1];   // dO rows
  __shared__ float Ls[kRows], Ds[kRows];
  const int b = blockIdx.z, g = blockIdx.y;
  const int key = threadIdx.x / kSub, sub = threadIdx.x % kSub;
  const int k0 = blockIdx.x * kRows;
  const int j = k0 + key;
  const bool valid = j < S;
  const int64_t krow = ((static_cast<int64_t>(b) * Hkv + g) * S + j) * D;
  const float scale = rsqrtf(static_cast<float>(D));
  float kr[DS], vr[DS], dka[DS], dva[DS];
#pragma unroll
  for (int i = 0; i < DS; ++i) {
    kr[i] = valid ? to_f32(k[krow + sub + kSub * i]) : 0.f;
    vr[i] = valid ? to_f32(v[krow + sub + kSub * i]) : 0.f;
    dka[i] = 0.f;
    dva[i] = 0.f;
  }
  auto dot4 = [&](const float (&a)[DS], const float* row_s) {
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < DS; ++i) part = fmaf(a[i], row_s[sub + kSub * i], part);
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    part += __shfl_xor_sync(0xffffffffu, part, 2);
    return part;
  };
  const int t_lo = causal ? k0 : 0;
  for (int hl = 0; hl < G; ++hl) {
    const int h = g * G + hl;
    for (int t0 = t_lo; t0 < S; t0 += kRows) {
      __syncthreads();
      for (int idx = threadIdx.x; idx < kRows * D; idx += kRows * kSub) {
        const int r = idx / D, c = idx % D;
        const int t = t0 + r;
        const int64_t qr = ((static_cast<int64_t>(b) * S + t) * Hq + h) * D + c;
        Qs[r][c] = t < S ? to_f32(q[qr]) * scale : 0.f;
        Os[r][c] = t < S ? to_f32(dout[qr]) : 0.f;
      }
      if (threadIdx.x < kRows) {
        const int t = t0 + threadIdx.x;
        const int64_t lr = (static_cast<int64_t>(b) * Hq + h) * S + t;
        Ls[threadIdx.x] = t < S ? lse_in[lr] : 0.f;
        Ds[threadIdx.x] = t < S ? dsum_in[lr] : 0.f;
      }
      __syncthreads();
      const int lim = min(kRows, S - t0);
      for (int r = 0; r < lim; ++r) {
        const float sc = dot4(kr, Qs[r]);
        const float dp = dot4(vr, Os[r]);
        const int t = t0 + r;
        if (!valid || (causal && j > t)) continue;
        const float p = expf(sc - Ls[r]);
        const float ds = p * (dp - Ds[r]);
#pragma unroll
        for (int i = 0; i < DS; ++i) {
          dva[i] = fmaf(p, Os[r][sub + kSub * i], dva[i]);
          dka[i] = fmaf(ds, Qs[r][sub + kSub * i], dka[i]);   // Qs holds q / sqrt(d)
        }
      }
    }
  }
  if (valid) {
#pragma unroll
    for (int i = 0; i < DS; ++i) {
      dk[krow + sub + kSub * i] = dka[i];
      dv[krow + sub + kSub * i] = dva[i];
    }
  }
}

// ----------------------------------------------------------------- rows
// One thread per (sequence, position, kv group, rotary pair i < d/2):
// RoPE transpose of dq and dk (turn back by the position's angle, taken modulo
// one turn in 64-bit fixed point as in the forward), the QK-mean transpose,
// and the value-shift transpose (a shifted channel of row t came from row
// t - 1, so row t's gradient there is row t + 1's).
template <typename T>
__global__ void rows_bwd_kernel(const BwdArgs<T> a) {
  const int d = a.d, half = d / 2, G = a.G;
  const int64_t total = static_cast<int64_t>(a.B) * a.S * a.Hkv * half;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int i = static_cast<int>(idx % half);
  int64_t rest = idx / half;
  const int g = static_cast<int>(rest % a.Hkv);
  rest /= a.Hkv;
  const int t = static_cast<int>(rest % a.S);
  const int b = static_cast<int>(rest / a.S);
  const int64_t row = static_cast<int64_t>(b) * a.S + t;
  float c = 1.f, s = 0.f;
  if (a.rope_on) {
    const uint64_t ph = static_cast<uint64_t>(t) * a.rope_frac[i];
    const float f = static_cast<float>(static_cast<int64_t>(ph)) * 5.42101086242752217e-20f;
    sincospif(2.0f * f, &s, &c);
  }
  // (lo, hi) was turned by +angle in the forward: its transpose turns by -angle
  auto unrot = [&](float lo, float hi, float& rlo, float& rhi) {
    rlo = lo * c + hi * s;
    rhi = hi * c - lo * s;
  };
  const int Cqk = (a.Hq + a.Hkv) * d;
  const int64_t kvrow = ((static_cast<int64_t>(b) * a.Hkv + g) * a.S + t) * d;
  float dkl, dkh;
  unrot(a.dk[kvrow + i], a.dk[kvrow + i + half], dkl, dkh);
  float sql = 0.f, sqh = 0.f;   // sum over the group's q heads of the unrotated dq
  for (int hl = 0; hl < G; ++hl) {
    const int h = g * G + hl;
    const int64_t qr = (row * a.Hq + h) * d;
    float ql, qh;
    unrot(a.dq[qr + i], a.dq[qr + i + half], ql, qh);
    sql += ql;
    sqh += qh;
    float yl = ql, yh = qh, ml = 0.f, mh = 0.f;
    if (a.qk_mean == 2) {
      yl *= 0.5f;
      yh *= 0.5f;
      ml = yl;
      mh = yh;
    } else if (a.qk_mean) {
      // m_q[h] = (q~[h] + k~[g]) / 2 and m_k[g] = (mean_h q~[h] + k~[g]) / 2
      ml = 0.5f * ql + (0.5f / G) * dkl;
      mh = 0.5f * qh + (0.5f / G) * dkh;
    }
    float* dy = a.dy + row * Cqk + h * d;
    float* dm = a.dzm + row * Cqk + h * d;
    dy[i] = yl;
    dy[i + half] = yh;
    dm[i] = ml;
    dm[i + half] = mh;
  }
  {
    float yl = dkl, yh = dkh, ml = 0.f, mh = 0.f;
    if (a.qk_mean == 2) {
      yl *= 0.5f;
      yh *= 0.5f;
      ml = yl;
      mh = yh;
    } else if (a.qk_mean) {
      ml = 0.5f * sql + 0.5f * dkl;
      mh = 0.5f * sqh + 0.5f * dkh;
    }
    float* dy = a.dy + row * Cqk + (a.Hq + g) * d;
    float* dm = a.dzm + row * Cqk + (a.Hq + g) * d;
    dy[i] = yl;
    dy[i + half] = yh;
    dm[i] = ml;
    dm[i + half] = mh;
  }
  // value-shift transpose into dz's v~ columns
  const bool next = t + 1 < a.S;
  const bool whole = a.value_shift == 2 && g >= a.Hkv - a.Hkv / 2;
  float* dzv = a.dz + row * a.N + (a.Hq + a.Hkv) * d + g * d;
  const float* dvt = a.dv + kvrow;
  const float* dvn = a.dv + kvrow + d;   // row t + 1 of the same sequence and group
  const float lo_cur = dvt[i], hi_cur = dvt[i + half];
  const float lo_nxt = next ? dvn[i] : 0.f, hi_nxt = next ? dvn[i + half] : 0.f;
  if (a.value_shift == 1) {
    dzv[i] = lo_cur;
    dzv[i + half] = hi_nxt;
  } else if (whole) {
    dzv[i] = lo_nxt;
    dzv[i + half] = hi_nxt;
  } else {
    dzv[i] = lo_cur;
    dzv[i + half] = hi_cur;
  }
}

// du = W^T dy per row and head (transpose of the per-position channel mix;
// du = dy for a side without one).  One thread per (row, head, channel j).
template <typename T>
__global__ void mix_bwd_kernel(const BwdArgs<T> a) {
  const int d = a.d, H = a.Hq + a.Hkv, Cqk = H * d;
  const int64_t total = static_cast<int64_t>(a.B) * a.S * Cqk;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int c = static_cast<int>(idx % Cqk);
  const int64_t row = idx / Cqk;
  const int head = c / d, j = c % d;
  const T* Wside = head < a.Hq ? a.wq_chan : a.wk_chan;
  const float* dy = a.dy + row * Cqk + head * d;
  if (!Wside) {
    a.du[row * Cqk + c] = dy[j];
    return;
  }
  const T* W = Wside + static_cast<int64_t>(head < a.Hq ? head : head - a.Hq) * d * d;
  float acc = 0.f;
  for (int ii = 0; ii < d; ++ii) acc = fmaf(to_f32(W[ii * d + j]), dy[ii], acc);
  a.du[row * Cqk + c] = acc;
}

// dz of the q~ and k~ columns: the QK-mean part plus the transpose of the conv.
// Depthwise: dz[t, c] += sum_j w[c, j] du[t + j, c]; temporal channel conv:
// dz[t, h, c] += sum_j sum_i W[h, j][i][c] dy[t + j, h, i]; no conv: dy.
// One thread per (row, channel).
template <typename T>
__global__ void conv_bwd_kernel(const BwdArgs<T> a) {
  const int d = a.d, H = a.Hq + a.Hkv, Cqk = H * d, K = a.K;
  const int64_t total = static_cast<int64_t>(a.B) * a.S * Cqk;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int c = static_cast<int>(idx % Cqk);
  const int64_t row = idx / Cqk;
  const int t = static_cast<int>(row % a.S);
  float acc = a.dzm[row * Cqk + c];
  if (K == 0) {
    acc += a.dy[row * Cqk + c];
  } else if (a.channel_conv) {
    const int head = c / d, cc = c % d;
    const T* W = head < a.Hq ? a.wq_chan + static_cast<int64_t>(head) * K * d * d
                             : a.wk_chan + static_cast<int64_t>(head - a.Hq) * K * d * d;
    for (int j = 0; j < K && t + j < a.S; ++j) {
      const float* dy = a.dy + (row + j) * Cqk + head * d;
      const T* Wj = W + static_cast<int64_t>(j) * d * d + cc;
      for (int ii = 0; ii < d; ++ii) acc = fmaf(to_f32(Wj[ii * d]), dy[ii], acc);
    }
  } else {
    const T* w = c < a.Hq * d ? a.wq_seq + static_cast<int64_t>(c) * K
                              : a.wk_seq + static_cast<int64_t>(c - a.Hq * d) * K;
    for (int j = 0; j < K && t + j < a.S; ++j) acc = fmaf(to_f32(w[j]), a.du[(row + j) * Cqk + c], acc);
  }
  a.dz[row * a.N + c] = acc;
}

// u = the depthwise conv of q~ / k~ (the channel mix's input), recomputed for
// the mix weights' gradient.  One thread per (row, channel).
template <typename T>
__global__ void conv_fwd_u_kernel(const BwdArgs<T> a) {
  const int d = a.d, Cqk = (a.Hq + a.Hkv) * d, K = a.K;
  const int64_t total = static_cast<int64_t>(a.B) * a.S * Cqk;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int c = static_cast<int>(idx % Cqk);
  const int64_t row = idx / Cqk;
  const int t = static_cast<int>(row % a.S);
  const T* w = c < a.Hq * d ? a.wq_seq + static_cast<int64_t>(c) * K
                            : a.wk_seq + static_cast<int64_t>(c - a.Hq * d) * K;
  float acc = 0.f;
  for (int j = 0; j < K && j <= t; ++j) acc = fmaf(to_f32(w[j]), to_f32(a.z[(row - j) * a.N + c]), acc);
  a.u[row * Cqk + c] = acc;
}

// Tap gradients: dw[c, j] = sum over (sequence, t >= j) of du[t, c] z[t - j, c].
// One thread per channel over a chunk of rows, atomically added.
template <typename T>
__global__ void tap_grad_kernel(const BwdArgs<T> a, int rows_per_chunk) {
  const int d = a.d, Cqk = (a.Hq + a.Hkv) * d, K = a.K;
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= Cqk) return;
  const int64_t rows = static_cast<int64_t>(a.B) * a.S;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_chunk;
  const int64_t r1 = min(rows, r0 + rows_per_chunk);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int64_t row = r0; row < r1; ++row) {
    const int t = static_cast<int>(row % a.S);
    const float g = a.du[row * Cqk + c];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (j < K && j <= t) acc[j] = fmaf(g, to_f32(a.z[(row - j) * a.N + c]), acc[j]);
  }
  float* dw = c < a.Hq * d ? a.g_q_seq + static_cast<int64_t>(c) * K
                           : a.g_k_seq + static_cast<int64_t>(c - a.Hq * d) * K;
  for (int j = 0; j < K; ++j) atomicAdd(dw + j, acc[j]);
}

// ----------------------------------------------------------------- GEMM
// C[z][m][n] (+)= sum_k A(m, k) B(k, n) in fp32 on the CUDA cores, with
// strided operands and a segmented k: the k-th term reads row
// (k / seg) * seg_stride + off + (k % seg) of each operand (off_a, off_b), so
// one call can sum over positions of several sequences with a shift.
struct GemmArgs {
  const void* A;
  const void* B;
  void* C;
  int M, N, K;
  int64_t sam, sak, sbk, sbn, scm, scn;
  int64_t bza, bzb, bzc;   // batch offsets (elements)
  int seg, seg_stride, off_a, off_b;
  int accumulate;
  int ksplit;              // -1: cut K into ranges whose partial sums are added atomically
                           // into C (fp32 C, zeroed by the caller); else one range
};
constexpr int kGBM = 64, kGBN = 64, kGBK = 16;

template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const GemmArgs g) {
  __shared__ float As[kGBK][kGBM + 1];
  __shared__ float Bs[kGBK][kGBN + 1];
  const int ks = g.ksplit > 1 ? g.ksplit : 1;
  const int bz = blockIdx.z / ks, kpart = blockIdx.z % ks;
  const TA* A = static_cast<const TA*>(g.A) + bz * g.bza;
  const TB* B = static_cast<const TB*>(g.B) + bz * g.bzb;
  TC* C = static_cast<TC*>(g.C) + bz * g.bzc;
  const int m0 = blockIdx.y * kGBM, n0 = blockIdx.x * kGBN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  // this CTA's K range: whole kGBK blocks, the last range takes the rest
  const int kblocks = (g.K + kGBK - 1) / kGBK;
  const int per = (kblocks + ks - 1) / ks;
  const int k_begin = kpart * per * kGBK;
  const int k_end = min(g.K, (kpart + 1) * per * kGBK);
  float acc[4][4] = {};
  for (int k0 = k_begin; k0 < k_end; k0 += kGBK) {
    for (int idx = threadIdx.x; idx < kGBK * kGBM; idx += 256) {
      const int kk = idx / kGBM, mm = idx % kGBM;
      const int k = k0 + kk, m = m0 + mm;
      float val = 0.f;
      if (k < k_end && m < g.M) {
        const int64_t r = static_cast<int64_t>(k / g.seg) * g.seg_stride + g.off_a + k % g.seg;
        val = to_f32(A[m * g.sam + r * g.sak]);
      }
      As[kk][mm] = val;
    }
    for (int idx = threadIdx.x; idx < kGBK * kGBN; idx += 256) {
      const int kk = idx / kGBN, nn = idx % kGBN;
      const int k = k0 + kk, n = n0 + nn;
      float val = 0.f;
      if (k < k_end && n < g.N) {
        const int64_t r = static_cast<int64_t>(k / g.seg) * g.seg_stride + g.off_b + k % g.seg;
        val = to_f32(B[r * g.sbk + n * g.sbn]);
      }
      Bs[kk][nn] = val;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGBK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) av[r] = As[kk][ty * 4 + r];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) bv[cc] = Bs[kk][tx * 4 + cc];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) acc[r][cc] = fmaf(av[r], bv[cc], acc[r][cc]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int m = m0 + ty * 4 + r;
    if (m >= g.M) continue;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int n = n0 + tx * 4 + cc;
      if (n >= g.N) continue;
      TC* p = C + m * g.scm + n * g.scn;
      float val = acc[r][cc];
      if constexpr (sizeof(TC) == 4) {
        if (ks > 1) {
          atomicAdd(reinterpret_cast<float*>(p), val);
          continue;
        }
      }
      if (g.accumulate) val += to_f32(*p);
      *p = from_f32<TC>(val);
    }
  }
}

template <typename TA, typename TB, typename TC>
cudaError_t gemm(GemmArgs g, int batch, cudaStream_t st) {
  if (g.seg <= 0) {
    g.seg = g.K > 0 ? g.K : 1;
    g.seg_stride = 0;
  }
  if (g.M <= 0 || g.N <= 0 || batch <= 0) return cudaSuccess;
  const int tiles = ((g.N + kGBN - 1) / kGBN) * ((g.M + kGBM - 1) / kGBM) * batch;
  if (sizeof(TC) == 4 && !g.accumulate && g.ksplit == -1) {
    // few output tiles over a long K (the weight gradients): split K so that
    // about two waves of CTAs run, each range at least 32 K blocks long; the
    // caller zeroed C, so the atomic sums start from zero
    int ks = (2 * sm_count() + tiles - 1) / tiles;
    const int max_ks = (g.K + 32 * kGBK - 1) / (32 * kGBK);
    if (ks > max_ks) ks = max_ks;
    g.ksplit = ks < 1 ? 1 : ks;
  }
  if (g.ksplit < 1) g.ksplit = 1;
  dim3 grid((g.N + kGBN - 1) / kGBN, (g.M + kGBM - 1) / kGBM, batch * g.ksplit);
  gemm_simt_kernel<TA, TB, TC><<<grid, 256, 0, st>>>(g);
  count_launches(1);
  return cudaGetLastError();
}

template <typename T>
__global__ void cast_kernel(const float* __restrict__ src, T* __restrict__ dst, int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = from_f32<T>(src[i]);
}

int blocks_for(int64_t n, int per) { return static_cast<int>((n + per - 1) / per); }

// out[c, r] = in[r, c] as bf16 for r < R, zero for R <= r < ldo (in: [R, C],
// leading dimension C; out: [C, ldo]).  32 x 32 tiles through shared memory.
template <typename TI>
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const TI* __restrict__ in,
                                                             bf16* __restrict__ out, int64_t R,
                                                             int64_t C, int64_t ldo) {
  __shared__ float tile[32][33];
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 32, c0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8 threads
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const int64_t r = r0 + ty + i, c = c0 + tx;
    tile[ty + i][tx] = (r < R && c < C) ? to_f32(in[r * C + c]) : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const int64_t c = c0 + ty + i, r = r0 + tx;
    if (c < C && r < ldo) out[c * ldo + r] = __float2bfloat16_rn(tile[tx][ty + i]);
  }
}

template <typename TI>
void transpose_bf16(const TI* in, bf16* out, int64_t R, int64_t C, int64_t ldo, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((C + 31) / 32), static_cast<unsigned>((ldo + 31) / 32));
  transpose_bf16_kernel<TI><<<grid, 256, 0, st>>>(in, out, R, C, ldo);
  count_launches(1);
}

template <typename T, int D>
cudaError_t launch_attn_bwd_d(const BwdArgs<T>& a, cudaStream_t st) {
  if constexpr (sizeof(T) == 2 && D >= 32) {
    if (a.o != nullptr && a.lse_ld > 0 && attn_bwd_tc_supported(D, a.G)) {
      // tensor core: the forward kernel recomputes o and the log-sum-exp, then
      // the dq pass and the dk / dv pass
      AttnArgs f{};
      f.q = a.q;
      f.k = a.k;
      f.v = a.v;
      f.out = a.o;
      f.B = a.B;
      f.S = a.S;
      f.Hq = a.Hq;
      f.Hkv = a.Hkv;
      f.d = D;
      f.G = a.G;
      f.kv_cap = a.S;
      f.causal = a.causal;
      f.dev_err = a.dev_err;
      f.lse = a.lse;
      f.lse_ld = a.lse_ld;
      cudaError_t e = launch_attn_prefill_tc(f, st);
      if (e != cudaSuccess) return e;
      AttnBwdTcArgs t{};
      t.q = a.q;
      t.k = a.k;
      t.v = a.v;
      t.o = a.o;
      t.dout = a.dout;
      t.lse = a.lse;
      t.dsum = a.dsum;
      t.ld = a.lse_ld;
      t.dq = a.dq;
      t.dk = a.dk;
      t.dv = a.dv;
      t.B = a.B;
      t.S = a.S;
      t.Hq = a.Hq;
      t.Hkv = a.Hkv;
      t.d = D;
      t.G = a.G;
      t.causal = a.causal;
      t.dev_err = a.dev_err;
      return launch_attn_bwd_tc(t, st);
    }
  }
  dim3 g1((a.S + kRows - 1) / kRows, a.Hq, a.B);
  attn_bwd_dq_kernel<T, D><<<g1, kRows * kSub, 0, st>>>(a.q, a.k, a.v, a.dout, a.dq, a.lse,
                                                         a.dsum, a.S, a.Hq, a.Hkv, a.G, a.causal);
  dim3 g2((a.S + kRows - 1) / kRows, a.Hkv, a.B);
  attn_bwd_dkdv_kernel<T, D><<<g2, kRows * kSub, 0, st>>>(a.q, a.k, a.v, a.dout, a.lse, a.dsum,
                                                           a.dk, a.dv, a.S, a.Hq, a.Hkv, a.G,
                                                           a.causal);
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace

template <typename T>
cudaError_t launch_backward(const BwdArgs<T>& a, cudaStream_t st) {
  cudaError_t e;
  switch (a.d) {
    case 16: e = launch_attn_bwd_d<T, 16>(a, st); break;
    case 32: e = launch_attn_bwd_d<T, 32>(a, st); break;
    case 64: e = launch_attn_bwd_d<T, 64>(a, st); break;
    case 128: e = launch_attn_bwd_d<T, 128>(a, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  const int d = a.d, H = a.Hq + a.Hkv, Cqk = H * d, K = a.K;
  const int64_t rows = static_cast<int64_t>(a.B) * a.S;
  rows_bwd_kernel<T><<<blocks_for(rows * a.Hkv * (d / 2), 256), 256, 0, st>>>(a);
  count_launches(1);
  const bool depthwise = K > 0 && !a.channel_conv;
  const bool mix = depthwise && (a.wq_chan || a.wk_chan);
  if (mix) {
    mix_bwd_kernel<T><<<blocks_for(rows * Cqk, 256), 256, 0, st>>>(a);
    count_launches(1);
  } else if (depthwise) {
    e = cudaMemcpyAsync(a.du, a.dy, static_cast<size_t>(rows) * Cqk * sizeof(float),
                        cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
  }
  conv_bwd_kernel<T><<<blocks_for(rows * Cqk, 256), 256, 0, st>>>(a);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // dx = dz W (or dz itself for packed input)
  bool gw_done = false;
  if constexpr (sizeof(T) == 2) {
    if (a.W && a.dz_b && a.WT && a.dzT && a.xT) {
      // tensor core: dx = bf16(dz) (W^T)^T, dW = bf16(dz)^T x as (dz^T)(x^T)^T
      cast_kernel<T><<<blocks_for(rows * a.N, 256), 256, 0, st>>>(a.dz, a.dz_b, rows * a.N);
      count_launches(1);
      transpose_bf16<T>(a.W, a.WT, a.N, a.E, a.N, st);
      if ((e = launch_proj_gemm_bf16(a.dz_b, a.WT, a.dx, static_cast<int>(rows), a.E, a.N,
                                     a.dev_err, st)) != cudaSuccess)
        return e;
      if (a.g_W) {
        transpose_bf16<float>(a.dz, a.dzT, rows, a.N, a.ldr, st);
        transpose_bf16<T>(a.x, a.xT, rows, a.E, a.ldr, st);
        if ((e = launch_gemm_bf16_f32out(a.dzT, a.xT, a.g_W, a.N, a.E, static_cast<int>(a.ldr),
                                         a.dev_err, st)) != cudaSuccess)
          return e;
      }
      gw_done = true;
    }
  }
  if (gw_done) {
  } else if (a.W) {
    GemmArgs g{};
    g.A = a.dz; g.B = a.W; g.C = a.dx;
    g.M = static_cast<int>(rows); g.N = a.E; g.K = a.N;
    g.sam = a.N; g.sak = 1; g.sbk = a.E; g.sbn = 1; g.scm = a.E; g.scn = 1;
    if ((e = gemm<float, T, T>(g, 1, st)) != cudaSuccess) return e;
  } else {
    cast_kernel<T><<<blocks_for(rows * a.N, 256), 256, 0, st>>>(a.dz, a.dx, rows * a.N);
    count_launches(1);
  }
  // weight gradients (each optional; the buffers were zeroed by the caller)
  if (a.g_W && a.W && !gw_done) {
    GemmArgs g{};
    g.A = a.dz; g.B = a.x; g.C = a.g_W;
    g.M = a.N; g.N = a.E; g.K = static_cast<int>(rows);
    g.sam = 1; g.sak = a.N; g.sbk = a.E; g.sbn = 1; g.scm = a.E; g.scn = 1;
    g.ksplit = -1;
    if ((e = gemm<float, T, float>(g, 1, st)) != cudaSuccess) return e;
  }
  if (depthwise && a.g_q_seq && a.g_k_seq) {
    const int chunk = 512;
    dim3 grid((Cqk + 127) / 128, static_cast<unsigned>((rows + chunk - 1) / chunk));
    tap_grad_kernel<T><<<grid, 128, 0, st>>>(a, chunk);
    count_launches(1);
  }
  if (mix && ((a.g_q_chan && a.wq_chan) || (a.g_k_chan && a.wk_chan))) {
    conv_fwd_u_kernel<T><<<blocks_for(rows * Cqk, 256), 256, 0, st>>>(a);
    count_launches(1);
    // dW_c[h][i][j] = sum over rows of dy[row, h d + i] u[row, h d + j]
    for (int side = 0; side < 2; ++side) {
      if (!(side ? (a.g_k_chan && a.wk_chan) : (a.g_q_chan && a.wq_chan))) continue;
      const int h0 = side ? a.Hq : 0, nh = side ? a.Hkv : a.Hq;
      GemmArgs g{};
      g.A = a.dy + h0 * d; g.B = a.u + h0 * d; g.C = side ? a.g_k_chan : a.g_q_chan;
      g.M = d; g.N = d; g.K = static_cast<int>(rows);
      g.sam = 1; g.sak = Cqk; g.sbk = Cqk; g.sbn = 1; g.scm = d; g.scn = 1;
      g.bza = d; g.bzb = d; g.bzc = static_cast<int64_t>(d) * d;
      g.ksplit = -1;
      if ((e = gemm<float, float, float>(g, nh, st)) != cudaSuccess) return e;
    }
  }
  if (K > 0 && a.channel_conv && a.g_q_chan && a.g_k_chan) {
    // dW[h, j][i][c] = sum over (sequence, t >= j) of dy[t, h, i] z[t - j, h, c]
    for (int side = 0; side < 2; ++side) {
      const int h0 = side ? a.Hq : 0, nh = side ? a.Hkv : a.Hq;
      for (int j = 0; j < K && j < a.S; ++j) {
        GemmArgs g{};
        g.A = a.dy + h0 * d; g.B = a.z + h0 * d;
        g.C = (side ? a.g_k_chan : a.g_q_chan) + static_cast<int64_t>(j) * d * d;
        g.M = d; g.N = d; g.K = a.B * (a.S - j);
        g.sam = 1; g.sak = Cqk; g.sbk = a.N; g.sbn = 1; g.scm = d; g.scn = 1;
        g.bza = d; g.bzb = d; g.bzc = static_cast<int64_t>(K) * d * d;
        g.seg = a.S - j; g.seg_stride = a.S; g.off_a = j; g.off_b = 0;
        g.ksplit = -1;
        if ((e = gemm<float, T, float>(g, nh, st)) != cudaSuccess) return e;
      }
    }
  }
  return cudaGetLastError();
}

template cudaError_t launch_backward<float>(const BwdArgs<float>&, cudaStream_t);
template cudaError_t launch_backward<bf16>(const BwdArgs<bf16>&, cudaStream_t);

}  // namespace ccgqa
