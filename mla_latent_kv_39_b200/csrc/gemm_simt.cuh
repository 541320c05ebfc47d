// Strided, batched GEMM on CUDA cores: C[b][m][n] = sum_k A[b][m][k] B[b][k][n].
// A and B each in their own type (storage type or fp32), accumulation in Acc
// (float, or double where the result must be the correctly rounded
// real-number dot product).  Used by the
// fp32 path for every projection and by the bf16 path where no tensor-core
// kernel applies.
#pragma once

#include "common.cuh"

namespace mla {

struct GemmSimtArgs {
  const void* A;
  const void* B;
  void* C;
  int M, N, K, batch;
  long long sAm, sAk, sAb;  // element strides of A along m, k, batch
  long long sBk, sBn, sBb;  // element strides of B along k, n, batch
  long long sCm, sCn, sCb;  // element strides of C (type Acc) along m, n, batch
};

constexpr int kSimtTile = 32;

// kAtomic: add the result into C with atomics instead of storing it (split-K
// partials summed in place; C must start at zero).
template <typename TA, typename TB, typename Acc, bool kAtomic = false>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmSimtArgs g) {
  __shared__ Acc As[kSimtTile][kSimtTile + 1];
  __shared__ Acc Bs[kSimtTile][kSimtTile + 1];
  const TA* A = static_cast<const TA*>(g.A) + (long long)blockIdx.z * g.sAb;
  const TB* B = static_cast<const TB*>(g.B) + (long long)blockIdx.z * g.sBb;
  Acc* C = static_cast<Acc*>(g.C) + (long long)blockIdx.z * g.sCb;
  const int m0 = blockIdx.y * kSimtTile, n0 = blockIdx.x * kSimtTile;
  const int tx = threadIdx.x % kSimtTile, ty = threadIdx.x / kSimtTile;  // ty in [0, 8)
  Acc acc[4] = {0, 0, 0, 0};
  for (int k0 = 0; k0 < g.K; k0 += kSimtTile) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = ty + 8 * r;
      const int m = m0 + row, kk = k0 + tx;
      As[row][tx] = (m < g.M && kk < g.K) ? (Acc)Store<TA>::ld(A + m * g.sAm + kk * g.sAk) : Acc(0);
      const int k = k0 + row, n = n0 + tx;
      Bs[row][tx] = (k < g.K && n < g.N) ? (Acc)Store<TB>::ld(B + k * g.sBk + n * g.sBn) : Acc(0);
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kSimtTile; ++k) {
      const Acc b = Bs[k][tx];
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[r] = fma(As[ty + 8 * r][k], b, acc[r]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int m = m0 + ty + 8 * r, n = n0 + tx;
    if (m < g.M && n < g.N) {
      if constexpr (kAtomic) atomicAdd(&C[m * g.sCm + n * g.sCn], acc[r]);
      else C[m * g.sCm + n * g.sCn] = acc[r];
    }
  }
}

template <typename TA, typename TB, typename Acc, bool kAtomic = false>
static cudaError_t gemm_simt(const GemmSimtArgs& g, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return cudaSuccess;
  dim3 grid((g.N + kSimtTile - 1) / kSimtTile, (g.M + kSimtTile - 1) / kSimtTile, g.batch);
  gemm_simt_kernel<TA, TB, Acc, kAtomic><<<grid, 256, 0, s>>>(g);
  note_launch();
  return cudaGetLastError();
}

// Row-major helpers ----------------------------------------------------------
// C[M,N] (Acc) = A[M,K] (row stride lda) x B[K,N] (row stride ldb)
template <typename TA, typename TB, typename Acc>
static cudaError_t gemm_rm(const void* A, long long lda, const void* B, long long ldb, Acc* C,
                           long long ldc, int M, int N, int K, cudaStream_t s) {
  GemmSimtArgs g{A, B, C, M, N, K, 1, lda, 1, 0, ldb, 1, 0, ldc, 1, 0};
  return gemm_simt<TA, TB, Acc>(g, s);
}

}  // namespace mla
