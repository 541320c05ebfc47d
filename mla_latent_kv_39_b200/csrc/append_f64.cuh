// Exact latent projection of the cache append on the fp64 pipe.
//
// "Multi-head Latent Attention (MLA) Nedir?" (yapayzekasozluk.tr), section
// "MLA nasıl çalışır?" (compression; decoupled RoPE), and "GQA, MQA ve MLA:
// attention KV cache'i nasıl belirler" (LLMScale), section "Multi-head latent
// attention (MLA)": every new token caches c_KV = x W_DKV and the small rotary
// key k_R = RoPE(x W_KR).  The cache is the bf16 rounding of the real-number
// product, so the sums are taken in fp64: a product of two bf16 (or fp32)
// values is exact in fp64, only the fp64 additions round, and one final
// rounding to bf16 then lands on the same value as rounding the exact sum
// (apart from ties closer than fp64 resolution).
//
// C[t][n] += sum_{k in chunk} x[t][k] * Wcat[k][n] with Wcat = [W_DKV | W_KR]
// taken column tile by column tile (a tile never straddles the two).  One CTA
// owns a 64-token x 64-column output tile and one K chunk (blockIdx.z); the
// chunks' fp64 sums meet in C by fp64 atomic adds (C starts at zero).
//
// The operands arrive as 16-byte cp.async copies into a three-stage ring of raw
// tiles, are widened to fp64 in shared memory once per tile, and each of the
// 128 threads then accumulates an 8 x 4 block of outputs (two k per step:
// 16-byte shared loads of fp64 pairs, 8 + 4 loads per 64 FMAs).
#pragma once

#include <atomic>

#include "common.cuh"

namespace mla {
namespace apf64 {

constexpr int BM = 64, BN = 64, BK = 32, kThreads = 128, kStages = 3;
constexpr int XS = BK + 2;  // fp64 row stride of the widened x tile (rows 16-byte aligned)

template <typename T>
struct Raw {
  T x[BM][BK];  // [token][k]
  T w[BK][BN];  // [k][column]
};

template <typename T>
struct Smem {
  Raw<T> raw[kStages];
  alignas(16) double xs[BM][XS];
  alignas(16) double ws[BK][BN];
};

template <typename T>
struct Args {
  const T* x;
  int ldx;
  const T* w_c;  // [hidden][d_c]
  int ld_c;
  const T* w_r;  // [hidden][d_r]
  int ld_r;
  int d_c;
  double* C;  // [M][ldC], columns [0, d_c + d_r) used
  int ldC;
  int M, Kc;  // tokens, K chunk per blockIdx.z (a multiple of BK)
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  const int n = valid ? 16 : 0;  // 0: fill the 16 bytes with zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ double2 widen2(const bf16* p) {
  const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(p);
  return make_double2((double)__bfloat162float(v.x), (double)__bfloat162float(v.y));
}
__device__ __forceinline__ double2 widen2(const float* p) {
  const float2 v = *reinterpret_cast<const float2*>(p);
  return make_double2((double)v.x, (double)v.y);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 2) append_f64_kernel(Args<T> a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem<T>& sm = *reinterpret_cast<Smem<T>*>(smem_raw);
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * BM, col0 = blockIdx.x * BN, k0 = blockIdx.z * a.Kc;
  const T* wbase;
  int ldw;
  if (col0 < a.d_c) {
    wbase = a.w_c + col0;
    ldw = a.ld_c;
  } else {
    wbase = a.w_r + (col0 - a.d_c);
    ldw = a.ld_r;
  }
  constexpr int V = 16 / sizeof(T);         // elements per 16-byte copy
  constexpr int CX = BK / V, CW = BN / V;   // copies per x row / per w row

  auto load = [&](int kt, int buf) {
    const int kk = k0 + kt * BK;
    Raw<T>& r = sm.raw[buf];
    for (int c = tid; c < BM * CX; c += kThreads) {
      const int row = c / CX, j = c % CX, m = m0 + row;
      const bool ok = m < a.M;
      cp_async16(&r.x[row][j * V], a.x + (long long)(ok ? m : 0) * a.ldx + kk + j * V, ok);
    }
    for (int c = tid; c < BK * CW; c += kThreads) {
      const int row = c / CW, j = c % CW;
      cp_async16(&r.w[row][j * V], wbase + (long long)(kk + row) * ldw + j * V, true);
    }
  };

  const int tx = tid % 16, ty = tid / 16;  // rows ty + 8i, columns 2tx + {0,1} + 32j
  double acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;

  const int KT = a.Kc / BK;
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < KT) load(s, s);
    cp_async_commit();
  }
  for (int kt = 0; kt < KT; ++kt) {
    cp_async_wait<kStages - 2>();  // this thread's copies of tile kt have landed
    __syncthreads();               // everyone's have; and tile kt-1 is fully consumed
    if (kt + kStages - 1 < KT) load(kt + kStages - 1, (kt + kStages - 1) % kStages);
    cp_async_commit();
    const Raw<T>& r = sm.raw[kt % kStages];
    for (int e = tid; e < BM * BK / 2; e += kThreads) {
      const int row = e / (BK / 2), j = 2 * (e % (BK / 2));
      *reinterpret_cast<double2*>(&sm.xs[row][j]) = widen2(&r.x[row][j]);
    }
    for (int e = tid; e < BK * BN / 2; e += kThreads) {
      const int row = e / (BN / 2), j = 2 * (e % (BN / 2));
      *reinterpret_cast<double2*>(&sm.ws[row][j]) = widen2(&r.w[row][j]);
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < BK; k += 2) {
      double2 xa[8], w0[2], w1[2];
#pragma unroll
      for (int i = 0; i < 8; ++i) xa[i] = *reinterpret_cast<const double2*>(&sm.xs[ty + 8 * i][k]);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        w0[j] = *reinterpret_cast<const double2*>(&sm.ws[k][2 * tx + 32 * j]);
        w1[j] = *reinterpret_cast<const double2*>(&sm.ws[k + 1][2 * tx + 32 * j]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          acc[i][2 * j] = fma(xa[i].x, w0[j].x, acc[i][2 * j]);
          acc[i][2 * j + 1] = fma(xa[i].x, w0[j].y, acc[i][2 * j + 1]);
          acc[i][2 * j] = fma(xa[i].y, w1[j].x, acc[i][2 * j]);
          acc[i][2 * j + 1] = fma(xa[i].y, w1[j].y, acc[i][2 * j + 1]);
        }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + ty + 8 * i;
    if (m >= a.M) continue;
    double* crow = a.C + (long long)m * a.ldC + col0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      atomicAdd(crow + 2 * tx + 32 * j, acc[i][2 * j]);
      atomicAdd(crow + 2 * tx + 32 * j + 1, acc[i][2 * j + 1]);
    }
  }
}

// ------------------------------------------------------------------ host side

// The tiled path needs 16-byte aligned operands and rows, whole column tiles
// on both weights and a hidden size made of whole K tiles.
template <typename T>
inline bool supports(const void* x, int ldx, const void* w_c, int ld_c, const void* w_r, int ld_r, int d_c,
                     int d_r, int hidden) {
  constexpr int V = 16 / sizeof(T);
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return al(x) && al(w_c) && al(w_r) && ldx % V == 0 && ld_c % V == 0 && ld_r % V == 0 && d_c % BN == 0 &&
         d_r % BN == 0 && hidden % BK == 0;
}

// K chunks: the largest split of the hidden size into whole K tiles (at least
// two per chunk) that still fits every CTA of the launch on the GPU at once
// (two per SM).
inline int choose_splits(int hidden, int tiles, int sms) {
  const int kb = hidden / BK;
  int best = 1;
  for (int S = 1; S <= kb; ++S)
    if (kb % S == 0 && kb / S >= 2 && (long long)tiles * S <= 2LL * sms) best = S;
  return best;
}

template <typename T>
inline cudaError_t launch(const Args<T>& a, int n_cols, int S, cudaStream_t s) {
  const size_t smem = sizeof(Smem<T>);
  static std::atomic<unsigned long long> attr_done{0};  // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !(attr_done.load() & (1ull << dev))) {
    e = cudaFuncSetAttribute(append_f64_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(1ull << dev);
  } else if (dev >= 64) {
    e = cudaFuncSetAttribute(append_f64_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const dim3 grid(n_cols / BN, (a.M + BM - 1) / BM, S);
  append_f64_kernel<T><<<grid, kThreads, smem, s>>>(a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace apf64
}  // namespace mla
