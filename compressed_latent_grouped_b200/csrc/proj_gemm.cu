// Latent down-projection x -> [q~ | k~ | v~]
// ("Compressed Convolutional Attention", Methodologie item 1: tokens are
// projected straight into the latent space of width E/C).
//
// bf16: C[M, N] = A[M, K] * W[N, K]^T on the 5th-generation tensor core.
//   One persistent CTA per SM walks 128 x 256 output tiles.  Warp 0 streams
//   128x64 A and 256x64 W tiles with TMA (128B swizzle) through a 4-stage
//   shared-memory ring; warp 1 allocates 2 x 256 TMEM columns and one thread
//   issues tcgen05.mma (M=128, N=256, K=16, fp32 accumulate) into them in turn;
//   warps 2-5 read a finished accumulator back with tcgen05.ld, 32 x 32 at a
//   time, into a swizzled staging buffer (two per warp, alternating; bf16, or
//   fp32 for the weight gradients of the backward pass) that a TMA tile store
//   writes out as whole output rows (clipped at M and N), while the next tile
//   accumulates into the other.
// fp32: a plain shared-memory tiled GEMM on the CUDA cores.
#include "kernels.h"
#include "sm100.cuh"

namespace ccgqa {
namespace {

using namespace sm100;

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kGemmThreads = 192;
constexpr uint32_t kATile = kBM * kBK * 2;      // 16 KB
constexpr uint32_t kBTile = kBN * kBK * 2;      // 32 KB
constexpr uint32_t kStageBytes = kATile + kBTile;
constexpr uint32_t kOffBar = kStages * kStageBytes;          // barriers, TMEM slot (< 1 KB)
constexpr uint32_t kOffOut = kOffBar + 1024;                  // output staging, 1024-aligned
// one 32 x 32 output chunk: bf16 rows of 64 B (64B swizzle), fp32 rows of 128 B
// (128B swizzle)
template <typename TC>
__host__ __device__ constexpr uint32_t out_buf() { return 32 * 32 * static_cast<uint32_t>(sizeof(TC)); }
template <typename TC>
constexpr size_t gemm_smem() { return size_t(kOffOut) + 4 * 2 * out_buf<TC>() + 1024; }  // + slack
static_assert(gemm_smem<float>() <= 232448, "fp32 staging exceeds shared memory");

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, const void* src, int c0,
                                             int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::
                   "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_addr(src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// at most one of this thread's bulk groups still reading shared memory
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// every bulk group of this thread complete
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Persistent: CTA c computes tiles c, c + gridDim.x, ... (tile t = row block
// t / n_tiles, column block t % n_tiles, so CTAs running together share A rows
// through L2).  The TMA ring and the k-block counter run on across tiles, and
// the accumulator alternates between two 256-column TMEM buffers, so the
// epilogue of one tile overlaps the main loop of the next.
template <typename TC>
__global__ void __launch_bounds__(kGemmThreads, 1)
    proj_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA,
                          const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmC, int M, int N, int K,
                          int32_t* dev_err) {
  pdl_enter();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;   // [2] accumulator b complete
  uint64_t* acc_empty = acc_full + 2;     // [2] accumulator b read back (128 arrivals)
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = (K + kBK - 1) / kBK;
  const int n_tiles = (N + kBN - 1) / kBN;
  const int tiles = n_tiles * ((M + kBM - 1) / kBM);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * kBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      int g = 0;   // k-blocks issued by this CTA so far
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const int m0 = (t / n_tiles) * kBM, n0 = (t % n_tiles) * kBN;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % kStages;
          if (!mbar_wait(&empty[s], ((g / kStages) & 1) ^ 1, &abort_flag, dev_err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          uint8_t* sa = smem + s * kStageBytes;
          tma_load_2d(sa, &tmA, &full[s], kb * kBK, m0);
          tma_load_2d(sa + kATile, &tmB, &full[s], kb * kBK, n0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(kBM, kBN, false);
      int g = 0, i = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++i) {
        const int bsel = i & 1;
        // the epilogue has read this accumulator's previous tile back
        if (!mbar_wait(&acc_empty[bsel], ((i >> 1) & 1) ^ 1, &abort_flag, dev_err)) break;
        tc_fence_after();
        const uint32_t acc = tmem + bsel * kBN;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % kStages;
          if (!mbar_wait(&full[s], (g / kStages) & 1, &abort_flag, dev_err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_addr(smem + s * kStageBytes);
          const uint32_t b_base = a_base + kATile;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            // K-major, 128B-swizzled tiles: 8-row groups 1024 B apart; a K step of
            // 16 bf16 advances the start address by 32 B inside the swizzle row.
            const uint64_t ad = make_smem_desc(a_base + k * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd = make_smem_desc(b_base + k * 32, 16, 1024, kSwizzle128B);
            mma_ss(acc, ad, bd, idesc, (kb | k) != 0);
          }
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&acc_full[bsel]);
      }
    }
  } else {
    // Epilogue: warp w may only touch TMEM lanes [32 (w % 4), 32 (w % 4) + 32).
    const int q4 = warp & 3;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    constexpr uint32_t kOutBuf = out_buf<TC>();
    uint8_t* stage = smem + kOffOut + (warp - 2) * 2 * kOutBuf;
    int i = 0, nst = 0;   // tiles read back, chunks stored by this warp
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int bsel = i & 1;
      if (!mbar_wait(&acc_full[bsel], (i >> 1) & 1, &abort_flag, dev_err)) break;
      tc_fence_after();
      const int m0 = (t / n_tiles) * kBM, n0 = (t % n_tiles) * kBN;
      const int r0 = m0 + q4 * 32;   // this warp's 32 output rows
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        const int col0 = n0 + c * 32;
        if (col0 >= N) break;  // warp-uniform
        uint32_t r[32];
        tmem_ld32(trow + bsel * kBN + c * 32, r);
        tmem_wait_ld();
        if (r0 >= M) continue;   // rows past M: nothing to store (warp-uniform)
        uint8_t* buf = stage + (nst & 1) * kOutBuf;
        if (nst >= 2) {
          // the store issued from this buffer two chunks ago has read it
          if (lane == 0) bulk_wait_read_1();
          __syncwarp();
        }
        if constexpr (sizeof(TC) == 4) {
#pragma unroll
          for (int v = 0; v < 8; ++v)
            *reinterpret_cast<uint4*>(buf + swz_offset(lane, v * 16, 128)) =
                make_uint4(r[v * 4], r[v * 4 + 1], r[v * 4 + 2], r[v * 4 + 3]);
        } else {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 pk;
            uint32_t* pw = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[v * 8 + 2 * e]),
                                                        __uint_as_float(r[v * 8 + 2 * e + 1]));
              pw[e] = *reinterpret_cast<uint32_t*>(&h2);
            }
            *reinterpret_cast<uint4*>(buf + swz_offset(lane, v * 16, 64)) = pk;
          }
        }
        fence_proxy_async_smem();   // the TMA unit reads what the threads wrote
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmC, buf, col0, r0);
          bulk_commit();
        }
        ++nst;
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[bsel]);
    }
    if (lane == 0) bulk_wait_all();   // no store may still read this CTA's shared memory
  }

  if (abort_flag && warp == 1 && lane == 0) {
    // Do not release TMEM while an MMA might still write it.
    mma_commit(drain);
    const long long t0 = clock64();
    while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitLimitCycles) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kBN);
  }
}

// ------------------------------------------------------------------ fp32 SIMT
constexpr int kFBM = 64, kFBN = 64, kFBK = 16;

__global__ void __launch_bounds__(256)
    proj_gemm_f32_kernel(const float* __restrict__ A, const float* __restrict__ W,
                         float* __restrict__ C, int M, int N, int K) {
  __shared__ float As[kFBK][kFBM + 4];
  __shared__ float Ws[kFBK][kFBN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * kFBM, n0 = blockIdx.x * kFBN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kFBK) {
    for (int i = threadIdx.x; i < kFBM * kFBK; i += 256) {
      const int r = i / kFBK, c = i % kFBK;
      const int gm = m0 + r, gk = k0 + c;
      As[c][r] = (gm < M && gk < K) ? A[static_cast<int64_t>(gm) * K + gk] : 0.f;
      const int gn = n0 + r;
      Ws[c][r] = (gn < N && gk < K) ? W[static_cast<int64_t>(gn) * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kFBK; ++k) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[k][ty * 4 + i];
        w[i] = Ws[k][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn < N) C[static_cast<int64_t>(gm) * N + gn] = acc[i][j];
    }
  }
}

}  // namespace

namespace {
template <typename TC>
cudaError_t launch_tc_gemm(const bf16* A, const bf16* W, TC* C, int M, int N, int K,
                           int32_t* dev_err, cudaStream_t stream) {
  constexpr bool f32 = sizeof(TC) == 4;
  CUtensorMap tmA, tmB, tmC;
  const uint64_t dA[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
  const uint64_t sA[1] = {static_cast<uint64_t>(K) * 2};
  const uint32_t bA[2] = {kBK, kBM};
  const uint64_t dB[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N)};
  const uint32_t bB[2] = {kBK, kBN};
  // 16-byte output row pitch for the TMA store
  if (N % (f32 ? 4 : 8) != 0) return cudaErrorInvalidValue;
  const uint64_t dC[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(M)};
  const uint64_t sC[1] = {static_cast<uint64_t>(N) * sizeof(TC)};
  const uint32_t bC[2] = {32, 32};
  if (!encode_tensor_map(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, dA, sA, bA,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, dB, sA, bB,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&tmC, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                         2, C, dC, sC, bC, f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(proj_gemm_bf16_kernel<TC>),
                             static_cast<int>(gemm_smem<TC>()));
  if (e != cudaSuccess) return e;
  const int sms = sm_count();
  const int tiles = ((N + kBN - 1) / kBN) * ((M + kBM - 1) / kBM);
  const int grid = tiles < sms ? tiles : sms;   // one persistent CTA per SM
  const cudaError_t el = launch_pdl(proj_gemm_bf16_kernel<TC>, dim3(grid), dim3(kGemmThreads),
                                    gemm_smem<TC>(), stream, tmA, tmB, tmC, M, N, K, dev_err);
  count_launches(1);
  return el != cudaSuccess ? el : cudaGetLastError();
}
}  // namespace

cudaError_t launch_proj_gemm_bf16(const bf16* A, const bf16* W, bf16* C, int M, int N, int K,
                                  int32_t* dev_err, cudaStream_t stream) {
  return launch_tc_gemm<bf16>(A, W, C, M, N, K, dev_err, stream);
}

cudaError_t launch_gemm_bf16_f32out(const bf16* A, const bf16* W, float* C, int M, int N, int K,
                                    int32_t* dev_err, cudaStream_t stream) {
  return launch_tc_gemm<float>(A, W, C, M, N, K, dev_err, stream);
}

cudaError_t launch_proj_gemm_f32(const float* A, const float* W, float* C, int M, int N, int K,
                                 cudaStream_t stream) {
  dim3 grid((N + kFBN - 1) / kFBN, (M + kFBM - 1) / kFBM);
  proj_gemm_f32_kernel<<<grid, 256, 0, stream>>>(A, W, C, M, N, K);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ccgqa
