// Split combine folded into the W_UV projection (tcgen05 + TMEM + TMA).
//
// "MLA · latent KV, decoupled RoPE và matrix absorption" (openarchlab),
// section 1 "Định nghĩa": W_UV is absorbed on the output side, so head h's
// output is o_h = o_lat_h W_UV_h.  The split-KV decode leaves, per segment s
// of query row v, a normalised partial O_s,h and its log2-sum-exp; since
// W_UV_h is linear,
//   o_h[v] = sum_s w_s,h (O_s,h W_UV_h),   w_s,h = 2^(lse_s,h - M) / sum 2^(lse - M)
// over the segments of row v.  So the projection runs over the segments (the
// N side of the MMA, B = the bf16 partials straight from the decode
// workspace) and the merge happens on the fp32 accumulator in the epilogue:
// no fp32 latent output, no separate combine or conversion pass.
//
// One CTA per head (M = 128 output features of W_UV_h, K = d_c = 512 in 8
// blocks of 64, N = segments rounded up to 16, at most 512 as two MMAs of up
// to 256).  Roles (192 threads): warp 0 TMA, warp 1 TMEM + MMA issue, warps
// 2-5 the merge (one feature per thread = one TMEM lane), which writes the
// row's head output in bf16 [rows][H][v_head], the layout the W_O
// projection reads.
#pragma once

#include "decode_plan.cuh"
#include "sm100.cuh"

namespace mla {
namespace ocomb {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kABytes = 128 * 128;     // 128 features x 64 k (two 64 x 64 boxes)
constexpr int kRingBytes = 176 * 1024;
constexpr int kMaxStages = 8;
constexpr int kMaxN = 512;
constexpr int kVHead = 128;           // output features per head (the MMA M)

// B rows a stage holds: all N columns in one box, or two boxes of 256 rows.
__host__ __device__ constexpr int b_rows(int N) { return N <= 256 ? N : 512; }
__host__ __device__ constexpr int stage_bytes(int N) { return (kABytes + b_rows(N) * 128 + 1023) / 1024 * 1024; }
__host__ __device__ constexpr int num_stages(int N) {
  return kRingBytes / stage_bytes(N) < kMaxStages ? kRingBytes / stage_bytes(N) : kMaxStages;
}

struct Smem {
  uint8_t ring[kRingBytes];  // first member: 1024-byte aligned
  uint64_t full[kMaxStages], empty[kMaxStages];
  uint64_t acc_full;
  float w[kMaxN];            // merge weight of each segment for this CTA's head
  int row[kMaxN];            // query row of each segment
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory over the 227 KiB per-block limit");
// the output tile of the most rows a launch takes (rows <= segments <= kMaxN) fits the ring
static_assert(kMaxN * kVHead * 2 <= kRingBytes, "output staging larger than the ring");

struct Params {
  const void* ws;   // decode workspace (plan, log2-sum-exp, partial outputs)
  long long ws_bytes;
  int batch, n_q, H, d_c, v_head;
  int N;            // MMA columns: max segments rounded up to 16 (<= 512)
  bf16* oh;         // [rows][H][v_head]
};

__device__ __forceinline__ void set_abort(Smem& sm) { *(volatile int*)&sm.abort_flag = 1; }
__device__ __forceinline__ bool aborted(Smem& sm) { return *(volatile int*)&sm.abort_flag != 0; }

__global__ void __launch_bounds__(kThreads, 1)
    uv_combine_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                      const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x;
  const int nst = num_stages(p.N), KB = p.d_c / 64;
  const uint32_t sbytes = (uint32_t)stage_bytes(p.N);
  const int n0 = p.N < 256 ? p.N : 256, n1 = p.N - n0;  // columns of the two MMAs

  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&amap);
    prefetch_tensormap(&bmap);
    // W_UV is not written by the kernels before this one: warm L2 with this head's first blocks
    for (int kb = 0; kb < KB && kb < nst; ++kb) {
      asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(&amap), "r"(h * p.v_head),
                   "r"(kb * 64)
                   : "memory");
      asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(&amap),
                   "r"(h * p.v_head + 64), "r"(kb * 64)
                   : "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();  // the decode's partials and plan come from the kernels before
  pdl_trigger();

  const DecodeHeader* hd = ws_at<DecodeHeader>(p.ws, 0);
  const bool valid = hd->magic == kPlanMagic && hd->batch == p.batch && hd->n_q == p.n_q && hd->H == p.H &&
                     hd->d_c == p.d_c && hd->layout.total <= p.ws_bytes && hd->layout.part_elem == 2 &&
                     hd->num_segments <= p.N;
  if (!valid && h == 0 && threadIdx.x == 0) report(MLA_ERR_WORKSPACE, 1, p.batch, p.n_q);

  if (warp == 0) {
    if (lane == 0 && valid) {
      // ------------------------------------------------ TMA producer
      const uint32_t tx = (uint32_t)kABytes + (uint32_t)b_rows(p.N) * 128u;
      int kb = 0;
      for (; kb < KB && !aborted(sm); ++kb) {
        const int st = kb % nst;
        if (kb >= nst && !mbar_wait(&sm.empty[st], ((kb / nst) - 1) & 1, 100)) {
          set_abort(sm);
          break;
        }
        uint8_t* a = sm.ring + st * sbytes;
        uint8_t* b = a + kABytes;
        mbar_arrive_expect_tx(&sm.full[st], tx);
        tma_load_2d(a, &amap, h * p.v_head, kb * 64, &sm.full[st]);
        tma_load_2d(a + kABytes / 2, &amap, h * p.v_head + 64, kb * 64, &sm.full[st]);
        tma_load_3d(b, &bmap, kb * 64, h, 0, &sm.full[st]);
        if (n1 > 0) tma_load_3d(b + 256 * 128, &bmap, kb * 64, h, 256, &sm.full[st]);
      }
      // never leave a copy in flight into shared memory that is about to be released
      for (int kk = kb - nst < 0 ? 0 : kb - nst; kk < kb; ++kk) mbar_wait(&sm.full[kk % nst], (kk / nst) & 1, 101);
    }
  } else if (warp == 1) {
    if (lane == 0 && valid) {
      // ------------------------------------------------ MMA issuer
      // A (W_UV_h, MN-major): 64-feature chunks 8 KiB apart (LBO), 8 k-rows 1 KiB
      // apart (SBO), K step q at +2 KiB q.  B (partials, K-major): rows 128 B
      // apart, 8-row groups 1 KiB apart, K step q at +32 B q.
      const uint32_t idesc0 = idesc_bf16_f32(128, n0, 1, 0);
      const uint32_t idesc1 = idesc_bf16_f32(128, n1 > 0 ? n1 : 16, 1, 0);
      int kb = 0;
      for (; kb < KB; ++kb) {
        const int st = kb % nst;
        if (!mbar_wait(&sm.full[st], (kb / nst) & 1, 102)) {
          set_abort(sm);
          break;
        }
        tc_fence_after();
        const uint32_t a_s = smem_u32(sm.ring + st * sbytes), b_s = a_s + kABytes;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint64_t ad = smem_desc(a_s + 2048 * q, kABytes / 2, 1024, kSwizzle128B);
          mma_ss(tmem, ad, smem_desc(b_s + 32 * q, 16, 1024, kSwizzle128B), idesc0, (kb | q) ? 1u : 0u);
          if (n1 > 0)
            mma_ss(tmem + 256, ad, smem_desc(b_s + 256 * 128 + 32 * q, 16, 1024, kSwizzle128B), idesc1,
                   (kb | q) ? 1u : 0u);
        }
        mma_commit(&sm.empty[st]);
      }
      mma_commit(&sm.acc_full);
    }
  } else {
    // ------------------------------------------------ merge of each row's segments
    const int qw = warp & 3;
    const int f = qw * 32 + lane;  // feature of W_UV_h == TMEM lane
    const int tid = (warp - 2) * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
    const int rows = p.batch * p.n_q;
    const DecodeLayout L = hd->layout;
    const int nseg = valid ? hd->num_segments : 0;
    const int4* segs = ws_at<int4>(p.ws, L.off_seg);
    const int* sfirst = ws_at<int>(p.ws, L.off_seq_first);
    const int* snseg = ws_at<int>(p.ws, L.off_seq_nseg);
    const float* lse = ws_at<float>(p.ws, L.off_lse);
    // This head's log2-sum-exps and each segment's row, in one coalesced pass
    // (the MMAs run meanwhile) ...
    for (int s = tid; s < nseg; s += 128) {
      sm.w[s] = lse[(long long)s * p.H + h];
      sm.row[s] = segs[s].x;
    }
    __syncwarp();
    named_sync(1, 128);
    // ... then, one row per thread, its merge weights in place: the segments
    // of a row are contiguous and ordered (the RowMerge arithmetic, in order)
    for (int v = tid; v < rows; v += 128) {
      const int first = valid ? sfirst[v] : 0, n = valid ? snseg[v] : 0;
      float M = -INFINITY;
      for (int k = 0; k < n; ++k) M = fmaxf(M, sm.w[first + k]);
      float Z = 0.f;
      if (M != -INFINITY)
        for (int k = 0; k < n; ++k) Z += exp2f(sm.w[first + k] - M);
      const float invZ = M != -INFINITY ? 1.f / Z : 0.f;
      for (int k = 0; k < n; ++k) sm.w[first + k] = invZ > 0.f ? exp2f(sm.w[first + k] - M) * invZ : 0.f;
    }
    __syncwarp();
    named_sync(1, 128);
    bool ok = valid && __all_sync(0xffffffffu, mbar_wait(&sm.acc_full, 0, 103));
    if (valid && !ok) set_abort(sm);
    tc_fence_after();
    // Every load and MMA on the ring is over: it holds the head's output rows
    // as a bf16 tile [rows][v_head] (rows without a segment stay zero).
    bf16* stage = reinterpret_cast<bf16*>(sm.ring);
    for (int v = 0; v < rows; ++v) stage[v * kVHead + f] = __float2bfloat16_rn(0.f);
    int cur = -1;
    float acc = 0.f;
    for (int c0 = 0; ok && c0 < nseg; c0 += 32) {
      // the chunk's rows and weights, one segment per lane, handed round by
      // shuffles (no shared-memory load between the stores below)
      const int sl = c0 + lane;
      const int row_l = sl < nseg ? sm.row[sl] : -1;
      const float w_l = sl < nseg ? sm.w[sl] : 0.f;
      uint32_t d[32];
      tmem_ld32(tl + (uint32_t)c0, d);  // columns c0..c0+31 (the second MMA's start at 256)
      // every shuffle first (independent, pipelined), then a branch-free pass
      int vk[32];
      float wk[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        vk[k] = __shfl_sync(0xffffffffu, row_l, k);
        wk[k] = __shfl_sync(0xffffffffu, w_l, k);
      }
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const int v = vk[k];       // -1 past the last segment: no row change, nothing to add
        const bool next_row = v >= 0 && v != cur;
        if (next_row && cur >= 0) stage[cur * kVHead + f] = __float2bfloat16_rn(acc);
        acc = next_row ? 0.f : acc;
        cur = next_row ? v : cur;
        // a zero weight (also past the last segment): a never-written partial, skipped
        acc = wk[k] != 0.f ? fmaf(wk[k], __uint_as_float(d[k]), acc) : acc;
      }
    }
    if (cur >= 0) stage[cur * kVHead + f] = __float2bfloat16_rn(acc);
    __syncwarp();
    named_sync(1, 128);
    // the tile out with 16-byte stores: a row's 256 bytes from 16 neighbouring threads
    const long long rstride = (long long)p.H * kVHead;
    for (int i = tid; i < rows * (kVHead / 8); i += 128) {
      const int v = i / (kVHead / 8), c = i % (kVHead / 8);
      *reinterpret_cast<uint4*>(p.oh + v * rstride + (long long)h * kVHead + 8 * c) =
          *reinterpret_cast<const uint4*>(stage + v * kVHead + 8 * c);
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

// ================================================================ host side
inline bool supports(const mla_config* c, int max_segments) {
  return c->dtype == MLA_BF16 && c->v_head == kVHead && c->d_c % 64 == 0 && max_segments <= kMaxN;
}

inline mla_status make_maps(const void* W_UV, const void* ws, const DecodeLayout& L, const mla_config* c, int N,
                            CUtensorMap* a, CUtensorMap* b) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return MLA_ERR_CUDA;
  {  // W_UV [d_c, H v_head], MN-major boxes of 64 features x 64 k
    const cuuint64_t dims[2] = {(cuuint64_t)c->n_heads * c->v_head, (cuuint64_t)c->d_c};
    const cuuint64_t strides[1] = {(cuuint64_t)c->n_heads * c->v_head * 2};
    const cuuint32_t box[2] = {64, 64};
    const cuuint32_t es[2] = {1, 1};
    if (enc(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W_UV), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  {  // partials [segments][H][d_c] bf16, boxes of 64 k x 1 head x up to 256 segments
    void* base = static_cast<char*>(const_cast<void*>(ws)) + L.off_o;
    const cuuint64_t dims[3] = {(cuuint64_t)c->d_c, (cuuint64_t)c->n_heads, (cuuint64_t)L.max_segments};
    const cuuint64_t strides[2] = {(cuuint64_t)c->d_c * 2, (cuuint64_t)c->n_heads * c->d_c * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)(N < 256 ? N : 256)};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc(b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

inline mla_status launch(const mla_config* c, const void* W_UV, const void* ws, size_t ws_bytes,
                         const DecodeLayout& L, bf16* oh, cudaStream_t s) {
  const int N = (L.max_segments + 15) / 16 * 16;
  if (N > kMaxN || (N > 256 && N - 256 > 256)) return MLA_ERR_UNSUPPORTED;
  CUtensorMap a, b;
  const mla_status ms = make_maps(W_UV, ws, L, c, N, &a, &b);
  if (ms != MLA_OK) return ms;
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (!bit || !(done.load(std::memory_order_acquire) & bit)) {
    if (cudaFuncSetAttribute(uv_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
        cudaSuccess)
      return MLA_ERR_CUDA;
    if (bit) done.fetch_or(bit, std::memory_order_acq_rel);
  }
  const Params p{ws, (long long)ws_bytes, L.batch, L.n_q, c->n_heads, c->d_c, c->v_head, N, oh};
  return launch_chained(uv_combine_kernel, dim3(c->n_heads), dim3(kThreads), kSmemBytes, s, a, b, p) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

}  // namespace ocomb
}  // namespace mla
