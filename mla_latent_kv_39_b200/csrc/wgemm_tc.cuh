// Weight-streaming GEMM on the sm_100 tensor cores (tcgen05 + TMEM + TMA).
//
// C[g][t][f] = sum_k X[t][g][k] W_g[k][f] for the projections of the decode
// step, where the weights (hundreds of MB) dominate the bytes and the tokens
// are few (a decode batch).  So the MMA runs "swap AB": 128 output features
// of W are the M side (A operand), the tokens the N side (B operand, N <= 256),
// and the weights stream through shared memory once.  The K dimension is cut
// into S splits so that every SM streams its share; each (group, feature tile,
// split) writes an fp32 partial, and a separate pass sums the splits in a fixed
// order (deterministic results) and applies the step's epilogue.
//
// A (weights, bf16) comes in two layouts:
//   MN-major: W stored [K, F] (features contiguous)  -> two 64-feature TMA boxes
//   K-major : W stored [F, K] (K contiguous; W_UK)    -> one 128-row TMA box
// B (activations, bf16, K contiguous) is a 3-D view [tokens, groups, K]; with
// `split` a second view holds the bf16 remainder (lo) of fp32 activations and
// both are accumulated against the same weights.
//
// Roles (192 threads): warp 0 TMA, warp 1 TMEM allocation + MMA issue, warps
// 2-5 read the accumulator (two TMEM buffers of 256 columns, so the drain of
// one work item overlaps the MMAs of the next).
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace mla {
namespace wg {

using namespace sm100;

constexpr int kMaxStages = 12;
constexpr int kABytes = 128 * 128;            // 128 features x 64 k, bf16
// 144 KiB: 6 stages at N = 64 stream as fast as 12, and leave room on each SM
// for the append kernel, which runs beside the query projections.
constexpr int kRingBytes = 144 * 1024;        // stages of A + N x 64 (or 2 x N x 64) of B
constexpr int kThreads = 192;

// Stage size for an MMA N (1 KiB aligned for the swizzle atoms) and how many
// fit the ring: 6 stages at N = 64, 3 at N = 256.
__host__ __device__ constexpr int stage_bytes(int N, int split) {
  return (kABytes + N * 128 * (split ? 2 : 1) + 1023) / 1024 * 1024;
}
__host__ __device__ constexpr int num_stages(int N, int split) {
  return kRingBytes / stage_bytes(N, split) < kMaxStages ? kRingBytes / stage_bytes(N, split) : kMaxStages;
}

struct Smem {
  uint8_t ring[kRingBytes];  // first member: 1024-byte aligned
  uint64_t full[kMaxStages], empty[kMaxStages];
  uint64_t acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory over the 227 KiB per-block limit");

struct Params {
  int G, MT, KB, S;     // groups, 128-feature tiles per group, 64-k blocks per group, K splits
  int n_tok, N;         // tokens, MMA N (tokens rounded up to 16)
  int a_kmajor;         // A layout (see above)
  int a_g_stride;       // MN-major: feature offset per group; K-major: k offset per group
  int split;            // B has a lo part
  int F;                // features per group
  float* part;          // [S][n_tok][G][F] (S > 1)
  float* out_f32;       // with S == 1 the accumulator goes straight to the outputs
  bf16* out_hi;
  bf16* out_lo;
  long long o_ts, o_gs;  // output element (t, g, f) at t o_ts + g o_gs + f
};

// Work item -> (group, feature tile, K split).  Consecutive items (which run
// on consecutive CTAs at about the same time) take neighbouring columns of the
// weight matrix for the same K rows, so together they read whole DRAM pages
// instead of 128-byte pieces of many: feature tiles then groups for
// MN-major weights (columns g * F + 128 mt), groups first for K-major ones
// (columns g * Kg + k).
__device__ __forceinline__ void item_coords(const Params& p, int item, int& g, int& mt, int& kb0, int& kb1, int& s) {
  const int tiles = p.G * p.MT;
  s = item / tiles;
  const int c = item % tiles;
  if (p.a_kmajor) {
    mt = c / p.G;
    g = c % p.G;
  } else {
    g = c / p.MT;
    mt = c % p.MT;
  }
  kb0 = (int)((long long)s * p.KB / p.S);
  kb1 = (int)((long long)(s + 1) * p.KB / p.S);
}

__device__ __forceinline__ void set_abort(Smem& sm) { *(volatile int*)&sm.abort_flag = 1; }
__device__ __forceinline__ bool aborted(Smem& sm) { return *(volatile int*)&sm.abort_flag != 0; }

__global__ void __launch_bounds__(kThreads, 1)
    wgemm_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap_hi,
                 const __grid_constant__ CUtensorMap bmap_lo, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int items = p.G * p.MT * p.S;
  const uint32_t b_bytes = (uint32_t)p.N * 128u;
  const uint32_t stage_tx = (uint32_t)kABytes + b_bytes * (p.split ? 2u : 1u);
  const int nst = num_stages(p.N, p.split);
  const uint32_t sbytes = (uint32_t)stage_bytes(p.N, p.split);

  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], 128);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&amap);
    prefetch_tensormap(&bmap_hi);
    if (p.split) prefetch_tensormap(&bmap_lo);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp != 0) {  // activations and output buffers belong to the kernels before
    pdl_wait();
    pdl_trigger();
  }

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      auto load_a = [&](uint8_t* a, int g, int mt, int kb, uint64_t* bar) {
        if (p.a_kmajor) {
          tma_load_2d(a, &amap, g * p.a_g_stride + kb * 64, mt * 128, bar);
        } else {
          tma_load_2d(a, &amap, g * p.a_g_stride + mt * 128, kb * 64, bar);
          tma_load_2d(a + kABytes / 2, &amap, g * p.a_g_stride + mt * 128 + 64, kb * 64, bar);
        }
      };
      // The weights are not written by the kernels before this one: the first
      // item's first stages of W go out before the wait, their activations after.
      int pre = 0;
      if (blockIdx.x < items) {
        int g, mt, kb0, kb1, s;
        item_coords(p, blockIdx.x, g, mt, kb0, kb1, s);
        pre = min(nst, kb1 - kb0);
        for (int i = 0; i < pre; ++i) {
          mbar_arrive_expect_tx(&sm.full[i], stage_tx);
          load_a(sm.ring + i * sbytes, g, mt, kb0 + i, &sm.full[i]);
        }
      }
      pdl_wait();
      pdl_trigger();
      int k = 0;
      for (int item = blockIdx.x; item < items && !aborted(sm); item += gridDim.x) {
        int g, mt, kb0, kb1, s;
        item_coords(p, item, g, mt, kb0, kb1, s);
        for (int kb = kb0; kb < kb1; ++kb, ++k) {
          const int st = k % nst;
          if (k >= nst && !mbar_wait(&sm.empty[st], ((k / nst) - 1) & 1, 70)) {
            set_abort(sm);
            goto producer_drain;
          }
          uint8_t* a = sm.ring + st * sbytes;
          uint8_t* b = a + kABytes;
          if (k >= pre) {
            mbar_arrive_expect_tx(&sm.full[st], stage_tx);
            load_a(a, g, mt, kb, &sm.full[st]);
          }
          tma_load_3d(b, &bmap_hi, kb * 64, g, 0, &sm.full[st]);
          if (p.split) tma_load_3d(b + b_bytes, &bmap_lo, kb * 64, g, 0, &sm.full[st]);
        }
      }
    producer_drain:
      // no copy may be in flight when the CTA leaves (the weight stages issued
      // before the wait included; a stage without its activations lands its
      // weights long before this bounded wait gives up)
      if (k < pre) k = pre;
      for (int kk = k - nst < 0 ? 0 : k - nst; kk < k; ++kk)
        mbar_wait(&sm.full[kk % nst], (kk / nst) & 1, 71);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16_f32(128, p.N, p.a_kmajor ? 0 : 1, 0);
      // A: MN-major -> 64-feature chunks 8 KiB apart (LBO), 8 k-rows 1 KiB apart
      // (SBO), K step j at +2 KiB * j; K-major -> rows 128 B apart, 8-row groups
      // 1 KiB apart (SBO), K step j at +32 B * j.  B: K-major like the latter.
      const uint64_t a0 = p.a_kmajor ? smem_desc(smem_u32(sm.ring), 16, 1024, kSwizzle128B)
                                     : smem_desc(smem_u32(sm.ring), kABytes / 2, 1024, kSwizzle128B);
      const uint64_t b0 = smem_desc(smem_u32(sm.ring) + kABytes, 16, 1024, kSwizzle128B);
      int k = 0, j = 0;
      for (int item = blockIdx.x; item < items; item += gridDim.x, ++j) {
        int g, mt, kb0, kb1, s;
        item_coords(p, item, g, mt, kb0, kb1, s);
        const int buf = j & 1;
        if (j >= 2 && !mbar_wait(&sm.acc_empty[buf], ((j >> 1) - 1) & 1, 72)) goto mma_fail;
        tc_fence_after();
        const uint32_t d = tmem + buf * 256;
        for (int kb = kb0; kb < kb1; ++kb, ++k) {
          const int st = k % nst;
          if (!mbar_wait(&sm.full[st], (k / nst) & 1, 73)) goto mma_fail;
          tc_fence_after();
          const uint32_t so = (st * sbytes) >> 4;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint64_t ad = a0 + so + ((p.a_kmajor ? q * 32u : q * 2048u) >> 4);
            const uint64_t bd = b0 + so + ((q * 32u) >> 4);
            mma_ss(d, ad, bd, idesc, (kb > kb0 || q > 0) ? 1u : 0u);
            if (p.split) mma_ss(d, ad, bd + (b_bytes >> 4), idesc, 1u);
          }
          mma_commit(&sm.empty[st]);
        }
        mma_commit(&sm.acc_full[buf]);
      }
      goto mma_end;
    mma_fail:
      set_abort(sm);
    mma_end:;
    }
  } else {
    // ------------------------------------------------ accumulator drain
    const int qw = warp & 3;
    const int f_local = qw * 32 + lane;  // feature within the 128-wide tile == TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
    int j = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x, ++j) {
      int g, mt, kb0, kb1, s;
      item_coords(p, item, g, mt, kb0, kb1, s);
      const int buf = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.acc_full[buf], (j >> 1) & 1, 74))) {
        set_abort(sm);
        break;
      }
      tc_fence_after();
      const long long tstride = (long long)p.G * p.F;
      const long long col = (long long)g * p.F + mt * 128 + f_local;
      const long long ocol = (long long)g * p.o_gs + mt * 128 + f_local;
      float* out = p.part + (long long)s * p.n_tok * tstride + col;
      for (int c = 0; c < p.N; c += 32) {
        uint32_t v[32];
        tmem_ld32(tl + buf * 256 + c, v);
        tmem_wait_ld();
        if (p.S > 1) {
#pragma unroll
          for (int t = 0; t < 32; ++t)
            if (c + t < p.n_tok) out[(long long)(c + t) * tstride] = __uint_as_float(v[t]);
        } else {  // one split: the step's outputs directly (a warp writes 32 consecutive features)
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            if (c + t >= p.n_tok) continue;
            const float x = __uint_as_float(v[t]);
            const long long o = (long long)(c + t) * p.o_ts + ocol;
            if (p.out_f32) p.out_f32[o] = x;
            if (p.out_hi) {
              const bf16 h = __float2bfloat16_rn(x);
              p.out_hi[o] = h;
              if (p.out_lo) p.out_lo[o] = __float2bfloat16_rn(x - __bfloat162float(h));
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.acc_empty[buf]);
    }
  }

  // The role branches above leave lanes of warps 0 and 1 apart (only lane 0
  // runs the producer or issuer loop): reconverge each warp before the
  // block-wide barrier, which counts whole warps.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

__device__ __forceinline__ void emit4(float4 v, long long i, float* out_f32, bf16* out_hi, bf16* out_lo) {
  if (out_f32) *reinterpret_cast<float4*>(out_f32 + i) = v;
  if (out_hi) {
    const float a[4] = {v.x, v.y, v.z, v.w};
    __align__(8) bf16 h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      h[e] = __float2bfloat16_rn(a[e]);
      l[e] = __float2bfloat16_rn(a[e] - __bfloat162float(h[e]));
    }
    *reinterpret_cast<uint2*>(out_hi + i) = *reinterpret_cast<const uint2*>(h);
    if (out_lo) *reinterpret_cast<uint2*>(out_lo + i) = *reinterpret_cast<const uint2*>(l);
  }
}

// out[t, g, f] = sum_s part[s][t][g][f] over `count` = n G F elements (F a
// multiple of 4), summed in split order, written as fp32 and/or bf16 (hi)
// and/or the bf16 remainder (lo = value - hi) at t o_ts + g o_gs + f.  Four
// elements per thread; the S loads of a group are issued before the adds so
// they are in flight together.
__global__ void reduce_splits_kernel(const float* __restrict__ part, int S, long long count, int G, int F,
                                     long long o_ts, long long o_gs, float* out_f32, bf16* out_hi, bf16* out_lo) {
  pdl_wait();
  pdl_trigger();
  constexpr int kBatch = 8;
  for (long long i = 4 * (blockIdx.x * (long long)blockDim.x + threadIdx.x); i < count;
       i += 4LL * gridDim.x * blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < S; s0 += kBatch) {
      float4 v[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b)
        if (s0 + b < S) v[b] = __ldcs(reinterpret_cast<const float4*>(part + (long long)(s0 + b) * count + i));
#pragma unroll
      for (int b = 0; b < kBatch; ++b)
        if (s0 + b < S) {
          acc.x += v[b].x;
          acc.y += v[b].y;
          acc.z += v[b].z;
          acc.w += v[b].w;
        }
    }
    const long long gf = (long long)G * F;
    const long long o = (i / gf) * o_ts + ((i / F) % G) * o_gs + i % F;
    emit4(acc, o, out_f32, out_hi, out_lo);
  }
}

// fp32 -> bf16 (hi) and optional remainder (lo); `count` a multiple of 4.
__global__ void split_bf16_kernel(const float* __restrict__ in, long long count, bf16* out_hi, bf16* out_lo) {
  pdl_wait();
  pdl_trigger();
  for (long long i = 4 * (blockIdx.x * (long long)blockDim.x + threadIdx.x); i < count;
       i += 4LL * gridDim.x * blockDim.x)
    emit4(__ldg(reinterpret_cast<const float4*>(in + i)), i, nullptr, out_hi, out_lo);
}

}  // namespace wg
}  // namespace mla

// ================================================================ host side
namespace mla {
namespace wg {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load(std::memory_order_acquire);
  if (f == nullptr) {
    void* q = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess && q != nullptr) {
      f = reinterpret_cast<EncodeTiledFn>(q);
      fn.store(f, std::memory_order_release);
    }
  }
  return f;
}

// One projection of the step: weights W (bf16, as stored) against bf16
// activations B[t][g][k] (element t * b_t_stride + g * b_g_stride + k).
struct Spec {
  const bf16* W;
  long long w_rows, w_cols;  // W as stored, row-major
  int a_kmajor;              // 0: W is [K, features]; 1: W is [features, K]
  int G, F, Kg;              // groups, features per group (x128), K per group (x64)
  int a_g_stride;            // MN-major: feature column offset of group g; K-major: k column offset
  const bf16* B_hi;
  const bf16* B_lo;          // optional bf16 remainder of fp32 activations
  long long b_t_stride, b_g_stride;
  int n_tok;                 // tokens of this call (<= 256)
  long long o_ts = 0, o_gs = 0;  // output strides (0: dense [n_tok][G][F])
};

inline long long out_ts(const Spec& s) { return s.o_ts ? s.o_ts : (long long)s.G * s.F; }
inline long long out_gs(const Spec& s) { return s.o_gs ? s.o_gs : s.F; }

inline bool spec_ok(const Spec& s) {
  return s.F % 128 == 0 && s.Kg % 64 == 0 && s.n_tok > 0 && s.G > 0;
}

// Tokens per launch: the MMA N is at most 256, and a stage holds 256 token
// rows of one activation view (128 rows each of hi and lo).
inline int max_chunk(const Spec& s) { return s.B_lo ? 128 : 256; }

// K splits.  The grid has min(items, SMs) CTAs and CTA c takes items c,
// c + grid, ...; the slowest CTA streams ceil(items / grid) items of about
// KB / S 16 KiB weight blocks each.  With S > 1 every split also writes an
// fp32 partial that a second kernel reads back (spread over all SMs, plus
// that launch, counted as 128 KiB).  Pick the S with the fewest bytes on the
// slowest SM, keeping the partials under a quarter of the weight bytes.
inline int choose_splits(const Spec& s, int sms) {
  const int MT = s.F / 128, KB = s.Kg / 64;
  const long long base = (long long)s.G * MT;
  const double wbytes = 2.0 * s.G * (double)s.F * s.Kg;
  const double out_bytes = 4.0 * s.G * (double)s.F * std::min(s.n_tok, max_chunk(s));
  int best = 1;
  double best_cost = -1.0;
  for (int S = 1; S <= KB; ++S) {
    if (S > 1 && S * out_bytes > 0.25 * wbytes) break;
    const long long items = base * S, grid = std::min<long long>(items, sms);
    double cost = (double)((items + grid - 1) / grid) * ((KB + S - 1) / S) * 16384.0;
    if (S > 1) cost += 2.0 * S * out_bytes / sms + 131072.0;
    if (best_cost < 0 || cost < best_cost) {
      best = S;
      best_cost = cost;
    }
  }
  return best;
}

inline size_t partial_floats(const Spec& s, int S) {
  return S > 1 ? (size_t)S * std::min(s.n_tok, max_chunk(s)) * s.G * s.F : 0;  // one split: no partials
}

inline int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return n > 0 ? n : 148;
}

inline mla_status make_maps(const Spec& s, int N, CUtensorMap* a, CUtensorMap* bh, CUtensorMap* bl) {
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return MLA_ERR_CUDA;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)s.w_cols, (cuuint64_t)s.w_rows};
    const cuuint64_t strides[1] = {(cuuint64_t)s.w_cols * 2};
    const cuuint32_t box[2] = {64, s.a_kmajor ? 128u : 64u};
    const cuuint32_t es[2] = {1, 1};
    if (enc(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void*)s.W, dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  const bf16* srcs[2] = {s.B_hi, s.B_lo};
  CUtensorMap* maps[2] = {bh, bl};
  for (int i = 0; i < 2; ++i) {
    const bf16* src = srcs[i] ? srcs[i] : s.B_hi;
    const cuuint64_t dims[3] = {(cuuint64_t)s.Kg, (cuuint64_t)s.G, (cuuint64_t)s.n_tok};
    const cuuint64_t strides[2] = {(cuuint64_t)(s.G > 1 ? s.b_g_stride : s.Kg) * 2, (cuuint64_t)s.b_t_stride * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)N};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc(maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void*)src, dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

inline mla_status set_attr() {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return MLA_OK;
  if (cudaFuncSetAttribute(wgemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return MLA_OK;
}

// Projection into fp32 partials [S][n_tok][G][F], then their sum into the
// requested outputs (fp32 and/or bf16 hi and/or bf16 lo), all [n_tok][G][F].
inline mla_status run(const Spec& s0, float* part, float* out_f32, bf16* out_hi, bf16* out_lo, cudaStream_t st) {
  if (!spec_ok(s0)) return MLA_ERR_UNSUPPORTED;
  const int chunk = max_chunk(s0);
  if (s0.n_tok > chunk) {
    for (int t0 = 0; t0 < s0.n_tok; t0 += chunk) {
      Spec c = s0;
      c.n_tok = std::min(chunk, s0.n_tok - t0);
      c.B_hi = s0.B_hi + (long long)t0 * s0.b_t_stride;
      c.B_lo = s0.B_lo ? s0.B_lo + (long long)t0 * s0.b_t_stride : nullptr;
      const long long o = (long long)t0 * out_ts(s0);
      const mla_status ms = run(c, part, out_f32 ? out_f32 + o : nullptr, out_hi ? out_hi + o : nullptr,
                                out_lo ? out_lo + o : nullptr, st);
      if (ms != MLA_OK) return ms;
    }
    return MLA_OK;
  }
  const Spec& s = s0;
  const int sms = device_sms();
  const int S = choose_splits(s, sms);
  const int N = (s.n_tok + 15) / 16 * 16;
  if (((uintptr_t)s.W & 15u) || ((uintptr_t)s.B_hi & 15u) || (s.B_lo && ((uintptr_t)s.B_lo & 15u)))
    return MLA_ERR_INVALID_ARG;
  CUtensorMap a, bh, bl;
  mla_status ms = make_maps(s, N, &a, &bh, &bl);
  if (ms != MLA_OK) return ms;
  if ((ms = set_attr()) != MLA_OK) return ms;
  Params p{s.G, s.F / 128, s.Kg / 64, S, s.n_tok, N, s.a_kmajor, s.a_g_stride, s.B_lo ? 1 : 0, s.F, part,
           out_f32, out_hi, out_lo, out_ts(s), out_gs(s)};
  const int items = s.G * (s.F / 128) * S;
  if (launch_chained(wgemm_kernel, dim3(std::min(items, sms)), dim3(kThreads), kSmemBytes, st, a, bh, bl, p) !=
      cudaSuccess)
    return MLA_ERR_CUDA;
  if (S == 1) return MLA_OK;
  const long long count = (long long)s.n_tok * s.G * s.F;
  const int blocks = (int)std::min<long long>((count / 4 + 255) / 256, 8 * sms);
  return launch_chained(reduce_splits_kernel, dim3(blocks), dim3(256), 0, st, (const float*)part, S, count, s.G, s.F,
                        out_ts(s), out_gs(s), out_f32, out_hi, out_lo) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

inline size_t run_partial_bytes(const Spec& s0) {
  if (!spec_ok(s0)) return 0;
  Spec s = s0;
  s.n_tok = std::min(s0.n_tok, max_chunk(s0));
  return partial_floats(s, choose_splits(s, device_sms())) * sizeof(float);
}

}  // namespace wg
}  // namespace mla
