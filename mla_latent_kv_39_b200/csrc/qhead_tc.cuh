// The absorbed query of one head in one kernel (tcgen05 + TMEM + TMA).
//
// "MLA · latent KV, decoupled RoPE và matrix absorption" (openarchlab),
// section 1 "Định nghĩa" (matrix absorption, decoupled RoPE) and "Multi-head
// Latent Attention (MLA) Nedir?" (yapayzekasozluk.tr), "MLA nasıl çalışır?"
// (query compression): for head h and token t, with c_Q = x W_DQ given,
//   q_nope = c_Q W_UQ[:, 192 h + (0..127)],  q_R = RoPE(c_Q W_UQ[:, 192 h + 128 + (0..63)], pos)
//   q_lat  = q_nope W_UK_h^T  (W_UK_h = W_UK[:, 128 h + (0..127)], d_c rows)
// and the decode's packed bf16 row [q_lat || q_R] (plus the bf16 remainders in
// split-query mode) is written directly.  One CTA per head and token chunk of
// up to 64 tokens: the first product streams the head's 192 columns of W_UQ
// (MN-major A, M = 128 per MMA: the 128 q_nope columns, and the 64 q_R columns
// over a zero second half), the epilogue rotates q_R and leaves q_nope in
// shared memory in bf16 as the K-major B operand of the second product, which
// streams W_UK_h (K-major A, four 128-row tiles of d_c).  This replaces the
// W_UQ projection over all heads, the fp32 round trip of q and its split
// launch, and the per-head W_UK projection.
//
// Rounding: fp32 accumulation over q_lora in order (no split of K), q_nope
// rounded to bf16 (hi, and lo = bf16(q - hi) in split-query mode), the
// rotation in fp64 from the fp32 q_R, rounded to fp32 and then to the packed
// bf16 (hi / lo), q_lat rounded to bf16 (hi / lo).  The fp32 mode (no packed
// rows) writes q_lat and the rotated q_R before those last roundings, which
// the decode then applies in the same way.
//
// Roles (192 threads): warp 0 TMA, warp 1 TMEM allocation and MMA issue,
// warps 2-5 the epilogues (one TMEM lane = one feature per thread).  The
// outputs are staged in shared memory as [64 tokens][64 columns] tiles and
// leave with bulk tensor stores.  Every wait is bounded (mbarriers only, no
// named barriers among the roles) and reports MLA_ERR_TIMEOUT.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace mla {
namespace qh {

using namespace sm100;

constexpr int kNope = 128, kRope = 64, kHeadCols = kNope + kRope, kDc = 512;
constexpr int kTok = 64;                 // tokens per CTA (the MMA N)
constexpr int kBox = 64 * 128;           // 64 rows x 128 bytes
constexpr int kRingBoxes = 20;           // 160 KiB of load stages, then of output tiles
constexpr int kOutTiles = kDc / 64 + 1;  // 64-column tiles of a packed row (q_lat, then q_R)
constexpr int kThreads = 192;
constexpr uint32_t kTmemNope = 0, kTmemRope = 64, kTmemLat = 128, kTmemCols = 512;
static_assert(2 * kOutTiles <= kRingBoxes, "output tiles (and remainders) must fit the ring");

// A stage holds the two 64-feature boxes of q_nope's columns of W_UQ, the
// q_R box and the c_Q box (and its remainder in split-query mode).
template <bool kSplit>
struct Ring {
  static constexpr int kStageBoxes = kSplit ? 5 : 4;
  static constexpr int kStages = kRingBoxes / kStageBoxes;
  static constexpr uint32_t kStageBytes = kStageBoxes * kBox;
};

struct Smem {
  uint8_t ring[kRingBoxes * kBox];  // first member: 1024-byte aligned
  uint8_t zero[kBox];               // the second (zero) half of the q_R A operand
  uint8_t qn[2][2][kBox];           // q_nope as B of the second product: [hi / lo][64-value K block]
  uint64_t full[5], empty[5], g1_done, q_ready, g2_done, out_ready;
  uint32_t tmem_base;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory over the 227 KiB per-block limit");

struct Params {
  int n_tok, H, kb1;        // tokens, heads, 64-value K blocks of c_Q
  const double* rot;        // [n_tok][kRope / 2][cos, sin]
  int packed;               // 1: bf16 packed rows through the output tensor maps; 0:
  float* q_lat;             // fp32 q_lat [n_tok][H][kDc] and
  float* q_rope;            // fp32 rotated q_R [n_tok][H][kRope]
  unsigned long long wait_ns;
};

__device__ __forceinline__ uint64_t kdesc(const void* p) { return smem_desc(smem_u32(p), 16, 1024, kSwizzle128B); }

template <bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
    qhead_kernel(const __grid_constant__ CUtensorMap uqmap, const __grid_constant__ CUtensorMap ukmap,
                 const __grid_constant__ CUtensorMap cqmap, const __grid_constant__ CUtensorMap cqlomap,
                 const __grid_constant__ CUtensorMap ohimap, const __grid_constant__ CUtensorMap olomap,
                 const Params p) {
  using R = Ring<kSplit>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, t0 = blockIdx.y * kTok;
  const int ntok = min(kTok, p.n_tok - t0);
  const uint64_t wns = p.wait_ns;

  for (int i = threadIdx.x; i < kBox / 16; i += kThreads) reinterpret_cast<uint4*>(sm.zero)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < R::kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.g1_done, 1);
    mbar_init(&sm.q_ready, 128);  // every epilogue thread
    mbar_init(&sm.g2_done, 1);
    mbar_init(&sm.out_ready, 128);
    fence_mbar_init();
  }
  fence_proxy_async_smem();  // the zero block is read by the tensor cores
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      prefetch_tensormap(&uqmap);
      prefetch_tensormap(&ukmap);
      prefetch_tensormap(&cqmap);
      if (kSplit) prefetch_tensormap(&cqlomap);
      // The weights do not depend on the kernels before: the first stages of
      // W_UQ go out before the wait for c_Q, and this head's W_UK slice is
      // pulled into L2 for the second product.
      const uint32_t cq_bytes = (kSplit ? 2u : 1u) * kBox;
      const int pre = min(R::kStages, p.kb1);
      for (int kb = 0; kb < pre; ++kb) {
        uint8_t* s = sm.ring + kb * R::kStageBytes;
        mbar_arrive_expect_tx(&sm.full[kb], 3u * kBox + cq_bytes);
        tma_load_2d(s, &uqmap, kHeadCols * h, 64 * kb, &sm.full[kb]);
        tma_load_2d(s + kBox, &uqmap, kHeadCols * h + 64, 64 * kb, &sm.full[kb]);
        tma_load_2d(s + 2 * kBox, &uqmap, kHeadCols * h + kNope, 64 * kb, &sm.full[kb]);
      }
      for (int mt = 0; mt < kDc / 128; ++mt)
        for (int kb = 0; kb < kNope / 64; ++kb) prefetch_l2_2d(&ukmap, kNope * h + 64 * kb, 128 * mt);
      pdl_wait();  // c_Q comes from the kernel before
      pdl_trigger();
      for (int kb = 0; kb < pre; ++kb) {
        uint8_t* s = sm.ring + kb * R::kStageBytes;
        tma_load_2d(s + 3 * kBox, &cqmap, 64 * kb, t0, &sm.full[kb]);
        if (kSplit) tma_load_2d(s + 4 * kBox, &cqlomap, 64 * kb, t0, &sm.full[kb]);
      }
      int k = pre;
      for (int kb = pre; kb < p.kb1; ++kb, ++k) {
        const int st = k % R::kStages;
        if (!mbar_wait(&sm.empty[st], ((k / R::kStages) - 1) & 1, 60, wns)) goto producer_done;
        uint8_t* s = sm.ring + st * R::kStageBytes;
        mbar_arrive_expect_tx(&sm.full[st], 3u * kBox + cq_bytes);
        tma_load_2d(s, &uqmap, kHeadCols * h, 64 * kb, &sm.full[st]);
        tma_load_2d(s + kBox, &uqmap, kHeadCols * h + 64, 64 * kb, &sm.full[st]);
        tma_load_2d(s + 2 * kBox, &uqmap, kHeadCols * h + kNope, 64 * kb, &sm.full[st]);
        tma_load_2d(s + 3 * kBox, &cqmap, 64 * kb, t0, &sm.full[st]);
        if (kSplit) tma_load_2d(s + 4 * kBox, &cqlomap, 64 * kb, t0, &sm.full[st]);
      }
      for (int mt = 0; mt < kDc / 128; ++mt)
        for (int kb = 0; kb < kNope / 64; ++kb, ++k) {
          const int st = k % R::kStages;
          if (k >= R::kStages && !mbar_wait(&sm.empty[st], ((k / R::kStages) - 1) & 1, 61, wns)) goto producer_done;
          mbar_arrive_expect_tx(&sm.full[st], 2u * kBox);
          tma_load_2d(sm.ring + st * R::kStageBytes, &ukmap, kNope * h + 64 * kb, 128 * mt, &sm.full[st]);
        }
    producer_done:
      // no copy may be in flight when the CTA leaves
      for (int kk = k - R::kStages < 0 ? 0 : k - R::kStages; kk < k; ++kk)
        mbar_wait(&sm.full[kk % R::kStages], (kk / R::kStages) & 1, 62, wns);
    }
  } else if (warp == 1) {
    pdl_wait();
    pdl_trigger();
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t id1 = idesc_bf16_f32(128, kTok, 1, 0);  // A MN-major (W_UQ columns), B K-major (c_Q)
      const uint32_t id2 = idesc_bf16_f32(128, kTok, 0, 0);  // A K-major (W_UK rows), B K-major (q_nope)
      int k = 0;
      bool ok = true;
      for (int kb = 0; kb < p.kb1 && ok; ++kb, ++k) {
        const int st = k % R::kStages;
        if (!(ok = mbar_wait(&sm.full[st], (k / R::kStages) & 1, 63, wns))) break;
        tc_fence_after();
        uint8_t* s = sm.ring + st * R::kStageBytes;
        // MN-major A: two 64-feature chunks LBO apart, 8 k-rows 1 KiB apart, K step 16 rows = 2 KiB
        const uint64_t an = smem_desc(smem_u32(s), kBox, 1024, kSwizzle128B);
        const uint64_t ar = smem_desc(smem_u32(s + 2 * kBox), smem_u32(sm.zero) - smem_u32(s + 2 * kBox), 1024,
                                      kSwizzle128B);
        const uint64_t bh = kdesc(s + 3 * kBox), bl = kdesc(s + 4 * kBox);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t acc = (kb > 0 || q > 0) ? 1u : 0u;
          mma_ss(tmem + kTmemNope, an + (q * 2048u >> 4), bh + (q * 32u >> 4), id1, acc);
          mma_ss(tmem + kTmemRope, ar + (q * 2048u >> 4), bh + (q * 32u >> 4), id1, acc);
          if (kSplit) {
            mma_ss(tmem + kTmemNope, an + (q * 2048u >> 4), bl + (q * 32u >> 4), id1, 1u);
            mma_ss(tmem + kTmemRope, ar + (q * 2048u >> 4), bl + (q * 32u >> 4), id1, 1u);
          }
        }
        mma_commit(&sm.empty[st]);
      }
      mma_commit(&sm.g1_done);
      if (ok) ok = mbar_wait(&sm.q_ready, 0, 64, wns);
      for (int mt = 0; mt < kDc / 128 && ok; ++mt)
        for (int kb = 0; kb < kNope / 64 && ok; ++kb, ++k) {
          const int st = k % R::kStages;
          if (!(ok = mbar_wait(&sm.full[st], (k / R::kStages) & 1, 65, wns))) break;
          tc_fence_after();
          const uint64_t a = kdesc(sm.ring + st * R::kStageBytes), qh = kdesc(sm.qn[0][kb]), ql = kdesc(sm.qn[1][kb]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            mma_ss(tmem + kTmemLat + mt * kTok, a + (q * 32u >> 4), qh + (q * 32u >> 4), id2, (kb > 0 || q > 0) ? 1u : 0u);
            if (kSplit) mma_ss(tmem + kTmemLat + mt * kTok, a + (q * 32u >> 4), ql + (q * 32u >> 4), id2, 1u);
          }
          mma_commit(&sm.empty[st]);
        }
      mma_commit(&sm.g2_done);
    }
  } else {
    // ------------------------------------------------ epilogues
    pdl_wait();  // the rotation table comes from the kernel before
    pdl_trigger();
    const int qw = warp & 3;
    const int f = qw * 32 + lane;                            // feature (TMEM lane)
    const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);  // this warp's lane quarter
    float rr[kTok];                                          // rotated q_R of feature f (f < 64)
    if (!__all_sync(0xffffffffu, mbar_wait(&sm.g1_done, 0, 66, wns))) goto epi_done;
    tc_fence_after();
    {
      // q_nope feature f of every token -> bf16 (hi / lo) at row t, column f
      // of the K-major B tiles (128-byte swizzle)
      uint8_t* hi_tile = sm.qn[0][f >> 6];
      uint8_t* lo_tile = sm.qn[1][f >> 6];
      const int c = f & 63;
#pragma unroll
      for (int half = 0; half < kTok / 32; ++half) {
        uint32_t v[32];
        tmem_ld32(tl + kTmemNope + 32 * half, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int t = 32 * half + j;
          const uint32_t off = (uint32_t)t * 128u + ((((uint32_t)c >> 3) ^ ((uint32_t)t & 7u)) << 4) + ((uint32_t)c & 7u) * 2u;
          const float x = __uint_as_float(v[j]);
          const bf16 hb = __float2bfloat16_rn(x);
          *reinterpret_cast<bf16*>(hi_tile + off) = hb;
          if (kSplit) *reinterpret_cast<bf16*>(lo_tile + off) = __float2bfloat16_rn(x - __bfloat162float(hb));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.q_ready);
    }
    if (qw < 2) {
      // q_R feature f (rows 64..127 of that product are zeros): rotate the
      // pair (2i, 2i + 1) by pos * theta^(-2i/d_r) in fp64.  Lanes f and f^1
      // share a pair: one loads its cosine, the other its sine.
      const int pr = f >> 1, odd = f & 1;
#pragma unroll
      for (int half = 0; half < kTok / 32; ++half) {
        double cr[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int t = 32 * half + j;
          cr[j] = t < ntok ? __ldg(p.rot + ((long long)(t0 + t) * (kRope / 2) + pr) * 2 + odd) : 0.0;
        }
        uint32_t v[32];
        tmem_ld32(tl + kTmemRope + 32 * half, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float x = __uint_as_float(v[j]);
          const float other = __shfl_xor_sync(0xffffffffu, x, 1);
          const double co = __shfl_xor_sync(0xffffffffu, cr[j], 1);
          const double cs = odd ? co : cr[j], sn = odd ? cr[j] : co;
          rr[32 * half + j] = odd ? (float)((double)other * sn + (double)x * cs)
                                  : (float)((double)x * cs - (double)other * sn);
        }
      }
      if (!p.packed) {
#pragma unroll
        for (int t = 0; t < kTok; ++t)
          if (t < ntok) p.q_rope[((long long)(t0 + t) * p.H + h) * kRope + f] = rr[t];
      }
    }
    if (!__all_sync(0xffffffffu, mbar_wait(&sm.g2_done, 0, 67, wns))) goto epi_done;
    tc_fence_after();
    if (p.packed) {
      // q_lat (and q_R) -> bf16 output tiles [64 tokens][64 columns] in the
      // ring (every load and MMA on it has completed), hi tiles 0..8, their
      // remainders 9..17, then out with bulk tensor stores
      const uint32_t col = (uint32_t)(f & 63) * 2u;
#pragma unroll 1
      for (int mt = 0; mt < kDc / 128; ++mt)
#pragma unroll 1
        for (int half = 0; half < kTok / 32; ++half) {
          uint32_t v[32];
          tmem_ld32(tl + kTmemLat + mt * kTok + 32 * half, v);
          tmem_wait_ld();
          uint8_t* hi = sm.ring + (2 * mt + (f >> 6)) * kBox + col;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const uint32_t off = (uint32_t)(32 * half + j) * 128u;
            const float x = __uint_as_float(v[j]);
            const bf16 hb = __float2bfloat16_rn(x);
            *reinterpret_cast<bf16*>(hi + off) = hb;
            if (kSplit) *reinterpret_cast<bf16*>(hi + kOutTiles * kBox + off) = __float2bfloat16_rn(x - __bfloat162float(hb));
          }
        }
      if (qw < 2) {
        uint8_t* hi = sm.ring + (kOutTiles - 1) * kBox + col;
#pragma unroll
        for (int t = 0; t < kTok; ++t) {
          const bf16 hb = __float2bfloat16_rn(rr[t]);
          *reinterpret_cast<bf16*>(hi + t * 128) = hb;
          if (kSplit) *reinterpret_cast<bf16*>(hi + kOutTiles * kBox + t * 128) = __float2bfloat16_rn(rr[t] - __bfloat162float(hb));
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&sm.out_ready);
      if (threadIdx.x == 64 && mbar_wait(&sm.out_ready, 0, 68, wns)) {
        for (int i = 0; i < kOutTiles; ++i) {
          tma_store_3d(&ohimap, sm.ring + i * kBox, 64 * i, h, t0);
          if (kSplit) tma_store_3d(&olomap, sm.ring + (kOutTiles + i) * kBox, 64 * i, h, t0);
        }
        bulk_commit_group();
        bulk_wait_read_all();
      }
    } else {
#pragma unroll 1
      for (int mt = 0; mt < kDc / 128; ++mt)
#pragma unroll 1
        for (int half = 0; half < kTok / 32; ++half) {
          uint32_t v[32];
          tmem_ld32(tl + kTmemLat + mt * kTok + 32 * half, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = 32 * half + j;
            if (t < ntok) p.q_lat[((long long)(t0 + t) * p.H + h) * kDc + 128 * mt + f] = __uint_as_float(v[j]);
          }
        }
    }
  epi_done:;
  }

  // The role branches above leave lanes of warps 0 and 1 apart (only lane 0
  // runs the producer or issuer loop): reconverge each warp before the
  // block-wide barrier, which counts whole warps.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// The fp64 rotation of every token's q_R pairs: rot[t][i] = (cos, sin) of
// pos[t] theta^(-2i/d_r), computed once per token and shared by all heads.
__global__ void rope_table_kernel(const int32_t* __restrict__ pos, int n_tok, double theta, double* __restrict__ rot) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_tok * (kRope / 2)) return;
  const int t = i / (kRope / 2), pr = i % (kRope / 2);
  double sn, cs;
  sincos((double)pos[t] * rope_inv_freq(theta, pr, kRope), &sn, &cs);
  rot[2 * i] = cs;
  rot[2 * i + 1] = sn;
}

// ================================================================ host side
// Up to this many tokens each head's weight columns are streamed once or
// twice (one CTA per head and 64 tokens); beyond, the batched projections
// reuse them better.
constexpr int kMaxTok = 128;

inline bool supports(const mla_config* c, int n_tok) {
  return c->dtype == MLA_BF16 && c->qk_nope == kNope && c->d_r == kRope && c->d_c == kDc && c->q_lora > 0 &&
         c->q_lora % 64 == 0 && n_tok > 0 && n_tok <= kMaxTok;
}

inline size_t rot_bytes(int n_tok) { return (size_t)n_tok * kRope * sizeof(double); }

// The per-token rotation table `rot` (rot_bytes(n) bytes of device scratch)
// that `launch` reads; it depends on the positions only, so it can be made
// before the kernels that produce c_Q.
inline mla_status launch_rope_table(const mla_config* c, int n, const int32_t* pos, double* rot, cudaStream_t s) {
  const int pairs = n * (kRope / 2);
  return launch_chained(rope_table_kernel, dim3((pairs + 255) / 256), dim3(256), 0, s, pos, n, c->rope_theta, rot) ==
                 cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

// q_packed (bf16 [n][H][d_c + d_r], + remainders in split-query mode), or
// with q_hi null the fp32 q_lat [n][H][d_c] and q_rope [n][H][d_r], from c_Q
// (bf16 [n][q_lora], + remainders), W_UQ [q_lora, H (nope + d_r)] and W_UK
// [d_c, H nope]; `rot` holds the table of launch_rope_table, ordered before.
inline mla_status launch(const mla_config* c, int n, const bf16* cq_hi, const bf16* cq_lo, const bf16* W_UQ,
                         const bf16* W_UK, const int32_t* pos, double* rot, bf16* q_hi, bf16* q_lo, float* q_lat,
                         float* q_rope, unsigned long long wait_ns, cudaStream_t s) {
  const bool split = (c->flags & MLA_FLAG_SPLIT_QUERY) != 0;
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return MLA_ERR_CUDA;
  const int H = c->n_heads;
  CUtensorMap uq, uk, cq, cql;
  const cuuint32_t es[2] = {1, 1};
  {  // W_UQ [q_lora][H (nope + d_r)]: boxes of 64 features x 64 k
    const cuuint64_t dims[2] = {(cuuint64_t)H * kHeadCols, (cuuint64_t)c->q_lora};
    const cuuint64_t str[1] = {(cuuint64_t)H * kHeadCols * 2};
    const cuuint32_t box[2] = {64, 64};
    if (enc(&uq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void*)W_UQ, dims, str, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  {  // W_UK [d_c][H nope]: boxes of 64 k x 128 rows
    const cuuint64_t dims[2] = {(cuuint64_t)H * kNope, (cuuint64_t)kDc};
    const cuuint64_t str[1] = {(cuuint64_t)H * kNope * 2};
    const cuuint32_t box[2] = {64, 128};
    if (enc(&uk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void*)W_UK, dims, str, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  const bf16* cqs[2] = {cq_hi, split ? cq_lo : cq_hi};
  CUtensorMap* cqm[2] = {&cq, &cql};
  for (int i = 0; i < 2; ++i) {  // c_Q [n][q_lora]: boxes of 64 k x 64 tokens (rows past n read as zero)
    const cuuint64_t dims[2] = {(cuuint64_t)c->q_lora, (cuuint64_t)n};
    const cuuint64_t str[1] = {(cuuint64_t)c->q_lora * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kTok};
    if (enc(cqm[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void*)cqs[i], dims, str, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_CUDA;
  }
  // packed rows [n][H][d_c + d_r] (and the remainders): boxes of 64 columns x
  // 1 head x 64 tokens (tokens past n are not written)
  CUtensorMap ohi = cq, olo = cq;
  if (q_hi != nullptr) {
    bf16* outs[2] = {q_hi, split ? q_lo : q_hi};
    CUtensorMap* om[2] = {&ohi, &olo};
    for (int i = 0; i < 2; ++i) {
      const cuuint64_t dims[3] = {(cuuint64_t)(kDc + kRope), (cuuint64_t)H, (cuuint64_t)n};
      const cuuint64_t str[2] = {(cuuint64_t)(kDc + kRope) * 2, (cuuint64_t)H * (kDc + kRope) * 2};
      const cuuint32_t box[3] = {64, 1, (cuuint32_t)kTok};
      const cuuint32_t es3[3] = {1, 1, 1};
      if (enc(om[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void*)outs[i], dims, str, box, es3,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return MLA_ERR_CUDA;
    }
  }
  auto kernel = split ? qhead_kernel<true> : qhead_kernel<false>;
  static std::atomic<uint64_t> attr{0};  // bit 2 dev + split: attribute set
  {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    const uint64_t bit = dev < 32 ? (1ull << (2 * dev + (split ? 1 : 0))) : 0ull;
    if (!(bit && (attr.load(std::memory_order_acquire) & bit))) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) != cudaSuccess)
        return MLA_ERR_CUDA;
      if (bit) attr.fetch_or(bit, std::memory_order_acq_rel);
    }
  }
  const Params p{n, H, c->q_lora / 64, rot, q_hi != nullptr ? 1 : 0, q_lat, q_rope, wait_ns};
  return launch_chained(kernel, dim3(H, (n + kTok - 1) / kTok), dim3(kThreads), kSmemBytes, s, uq, uk, cq, cql, ohi,
                        olo, p) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

}  // namespace qh
}  // namespace mla
