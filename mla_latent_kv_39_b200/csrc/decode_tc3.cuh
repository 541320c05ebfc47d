// Latent-space split-KV decode on the sm_100 tensor cores.
//
// "MLA · latent KV, decoupled RoPE và matrix absorption" (openarchlab),
// section 1 "Định nghĩa" and section 2 "Luồng": with W_UK absorbed into the
// query and W_UV into the output side, for every head h of query row v
//   s_t = q_lat[h] . c_t + q_R[h] . k_R,t          (t over the cached tokens)
//   o_lat[h] = sum_t softmax(scale * s)_t c_t        (the latent output)
// The split-KV plan hands every worker one contiguous run of pages (one or
// more query rows, "segments"); a worker writes, per segment, the normalised
// partial output and its log2-sum-exp, which the combine merges.
//
// Work split: each worker is served by two independent CTAs that stream the
// same pages (the second read hits L2).  CTA `half` computes the full scores
// of every page for all 128 heads and accumulates only its half of the
// latent output, O[:, 256 half + (0..255)].  The score work is done twice;
// that is cheaper on this part than exchanging partial scores between SMs,
// since SM-to-SM (distributed shared memory) traffic runs at roughly
// 35 GB/s per SM, about as slow as the SM's share of HBM bandwidth.
//
// Warp roles (224 threads): warp 0 issues the TMA page loads and L2
// prefetches; warp 1 issues the score MMAs; warp 2 the P V MMAs (one thread
// issues a tcgen05.mma only every ~55 cycles, so the two products get their
// own issuers and overlap in the tensor pipe); warps 3..6 run the online
// softmax, one head row per thread, and write the segment's partial output.
//
// TMEM (512 columns x 128 lanes, lane = head): [0,256) this CTA's O half;
// [256,384) the query's latent columns of the same half as bf16 pairs (the A
// operand of 16 of the 36 score K-steps); [384,448) and [448,512) two score
// tiles.  P (bf16) is written over the first 32 columns of the score tile it
// came from and read from there by the P V MMAs.
//
// Shared memory: two page slots.  A slot keeps apart the 5 slabs (64 tokens x
// 64 values, 128-byte swizzle) that only the score MMAs read - the other
// latent half and the rotary key - and the 4 value slabs of this CTA's half:
// the first group is released as soon as the page's scores are done, the
// second when its P V is done, so the next page of the slot starts loading
// early.  The query's other 320 columns (bf16, same swizzle) are the
// shared-memory A operand of the remaining 20 score K-steps.
//
// Every wait gives up after a time limit, records MLA_ERR_TIMEOUT and makes
// all roles wind down without leaving copies or MMAs in flight.
#pragma once

#include "decode_plan.cuh"
#include "sm100.cuh"

namespace mla {
namespace tcdec3 {

using namespace sm100;

constexpr int kH = 128, kDc = 512, kDr = 64, kBS = 64, kRow = kDc + kDr;
constexpr int kSlab = 64 * 128;    // 64 rows x 64 bf16, 128-byte swizzle
constexpr int kQSlab = 128 * 128;  // 128 rows x 64 bf16
constexpr int kEarly = 5, kVal = 4;
constexpr int kPrefetch = 6;       // pages prefetched into L2 ahead of the loads
constexpr int kTmemO = 0, kTmemQ = 256, kTmemS = 384, kTmemCols = 512;
constexpr int kSoftmaxWarps = 4;
constexpr int kThreads = 32 * (3 + kSoftmaxWarps);
constexpr float kRescaleLog2 = 8.f;

struct Smem {
  uint8_t early[2][kEarly][kSlab];  // first member: 1024-byte aligned
  uint8_t val[2][kVal][kSlab];
  uint8_t qs[kEarly][kQSlab];
  uint64_t early_full[2], val_full[2], early_free[2], val_free[2];
  uint64_t s_full[2], p_ready[2], pv_done[2];
  uint64_t q_full, q_ready, s_fin, pv_fin;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory over the 227 KiB per-block limit");

struct Params {
  const float* q_lat;   // [rows, 128, 512]
  const float* q_rope;  // [rows, 128, 64]
  const int32_t* block_table;
  const int32_t* seq_lens;
  int max_blocks, num_blocks, n_q;
  float scale_log2;
  void* ws;
  DecodeLayout L;
};

// Logical 64-column slab of the 576-wide row held in early slot i / value slot i.
__device__ __forceinline__ int early_slab(int half, int i) { return i < 4 ? 4 * (1 - half) + i : 8; }
__device__ __forceinline__ int val_slab(int half, int i) { return 4 * half + i; }

__device__ __forceinline__ void set_abort(Smem& sm) { *(volatile int*)&sm.abort_flag = 1; }
__device__ __forceinline__ bool aborted(Smem& sm) { return *(volatile int*)&sm.abort_flag != 0; }

__device__ __forceinline__ void prefetch_l2_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(map), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void prefetch_line(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Descriptors differ only in the start address (bits 0-13, 16-byte units).
__device__ __forceinline__ uint64_t desc_at(uint64_t d, uint32_t byte_offset) { return d + (byte_offset >> 4); }

// ---------------------------------------------------------------- pages
// Walks the worker's pages in order: (segment, page) -> physical block.
struct PageCursor {
  const int4* segs;
  int si, seg_end, blk;
  __device__ bool valid() const { return si < seg_end; }
  __device__ void next() {
    if (++blk >= segs[si].z) {
      if (++si < seg_end) blk = segs[si].y;
    }
  }
};

__device__ __forceinline__ int phys_block(const Params& p, const int4* segs, const PageCursor& c, bool report_err) {
  const int b = segs[c.si].x / p.n_q;
  int phys = p.block_table[(long long)b * p.max_blocks + c.blk];
  if (phys < 0 || phys >= p.num_blocks) {
    if (report_err) report(MLA_ERR_BOUNDS, 5, b, phys);
    phys = 0;  // keep the pipeline moving; the error word marks the result invalid
  }
  return phys;
}

// ---------------------------------------------------------------- TMA producer
__device__ void producer(Smem& sm, const CUtensorMap* tmap, const Params& p, int seg_begin, int seg_end,
                         int half) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  PageCursor cur{segs, seg_begin, seg_end, seg_begin < seg_end ? segs[seg_begin].y : 0};
  PageCursor ahead = cur;
  auto prefetch_page = [&](const PageCursor& c) {  // one CTA of the pair warms L2 for both
    if (half != 0) return;
    const int phys = phys_block(p, segs, c, false);
    for (int s = 0; s < kRow / 64; ++s) prefetch_l2_2d(tmap, s * 64, phys * kBS);
  };
  int ne = 0, nv = 0;  // pages whose early / value loads were issued
  int ai = 0;          // page index of `ahead`
  for (; cur.valid() && !aborted(sm); cur.next()) {
    const int k = ne, slot = k & 1;
    const uint32_t use = (uint32_t)k >> 1;
    const int phys = phys_block(p, segs, cur, true);
    if (k >= 2 && !mbar_wait(&sm.early_free[slot], (use - 1) & 1, 40)) {
      set_abort(sm);
      break;
    }
    mbar_arrive_expect_tx(&sm.early_full[slot], kEarly * kSlab);
    for (int i = 0; i < kEarly; ++i)
      tma_load_2d(sm.early[slot][i], tmap, early_slab(half, i) * 64, phys * kBS, &sm.early_full[slot]);
    ++ne;
    if (k >= 2 && !mbar_wait(&sm.val_free[slot], (use - 1) & 1, 41)) {
      set_abort(sm);
      break;
    }
    mbar_arrive_expect_tx(&sm.val_full[slot], kVal * kSlab);
    for (int i = 0; i < kVal; ++i)
      tma_load_2d(sm.val[slot][i], tmap, val_slab(half, i) * 64, phys * kBS, &sm.val_full[slot]);
    ++nv;
    // keep L2 warm kPrefetch pages ahead, growing the window by at most two
    // pages per loaded page (a start-up burst of prefetches from every CTA
    // would delay everyone's first pages)
    for (int n = 0; n < 2 && ai <= k + kPrefetch && ahead.valid(); ++ai, ahead.next())
      if (ai > k) {
        prefetch_page(ahead);
        ++n;
      }
  }
  // never leave a copy in flight into shared memory that is about to be released
  for (int kk = ne - 2 < 0 ? 0 : ne - 2; kk < ne; ++kk)
    mbar_wait(&sm.early_full[kk & 1], ((uint32_t)kk >> 1) & 1, 42);
  for (int kk = nv - 2 < 0 ? 0 : nv - 2; kk < nv; ++kk)
    mbar_wait(&sm.val_full[kk & 1], ((uint32_t)kk >> 1) & 1, 43);
}

// ---------------------------------------------------------------- score MMAs
__device__ void score_issuer(Smem& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  constexpr uint32_t idesc = idesc_bf16_f32(128, 64, 0, 0);
  // K-major, 128-byte swizzle: rows 128 B apart, 8-row groups 1 KiB apart;
  // K step j (16 values) starts 32 B further.
  const uint64_t qd = smem_desc(smem_u32(sm.qs[0]), 16, 1024, kSwizzle128B);
  const uint64_t ed = smem_desc(smem_u32(sm.early[0][0]), 16, 1024, kSwizzle128B);
  const uint64_t vd = smem_desc(smem_u32(sm.val[0][0]), 16, 1024, kSwizzle128B);
  int k = 0, seg_i = 0;
  for (int si = seg_begin; si < seg_end; ++si, ++seg_i) {
    const int T = segs[si].z - segs[si].y;
    if (!mbar_wait(&sm.q_ready, seg_i & 1, 50) || !mbar_wait(&sm.q_full, seg_i & 1, 49)) goto fail;
    for (int i = 0; i < T; ++i) {
      const int kk = k + i, slot = kk & 1;
      const uint32_t use = (uint32_t)kk >> 1;
      // the score tile still holds P of page kk - 2 until its P V is done
      if (kk >= 2 && !mbar_wait(&sm.pv_done[slot], (use - 1) & 1, 51)) goto fail;
      if (!mbar_wait(&sm.early_full[slot], use & 1, 52)) goto fail;
      tc_fence_after();
      const uint32_t d = tmem + kTmemS + slot * 64;
#pragma unroll
      for (int e = 0; e < kEarly; ++e)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_ss(d, desc_at(qd, e * kQSlab + j * 32), desc_at(ed, (slot * kEarly + e) * kSlab + j * 32), idesc,
                 (e | j) ? 1u : 0u);
      mma_commit(&sm.early_free[slot]);
      if (!mbar_wait(&sm.val_full[slot], use & 1, 53)) goto fail;
      tc_fence_after();
#pragma unroll
      for (int e = 0; e < kVal; ++e)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_ts(d, tmem + kTmemQ + (e * 4 + j) * 8, desc_at(vd, (slot * kVal + e) * kSlab + j * 32), idesc, 1u);
      mma_commit(&sm.s_full[slot]);
    }
    k += T;
  }
  mma_commit(&sm.s_fin);
  mbar_wait(&sm.s_fin, 0, 54);
  return;
fail:
  set_abort(sm);
  mma_commit(&sm.s_fin);
  mbar_wait(&sm.s_fin, 0, 55);
}

// ---------------------------------------------------------------- P V MMAs
__device__ void pv_issuer(Smem& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  constexpr uint32_t idesc = idesc_bf16_f32(128, 256, 0, 1);
  // Value slabs as an MN-major B operand: 64-value chunks 8 KiB apart (LBO),
  // 8-token groups 1 KiB apart (SBO); K step j (16 tokens) starts 2 KiB further.
  const uint64_t vd = smem_desc(smem_u32(sm.val[0][0]), kSlab, 1024, kSwizzle128B);
  int k = 0;
  for (int si = seg_begin; si < seg_end; ++si) {
    const int T = segs[si].z - segs[si].y;
    for (int i = 0; i < T; ++i) {
      const int kk = k + i, slot = kk & 1;
      if (!mbar_wait(&sm.p_ready[slot], ((uint32_t)kk >> 1) & 1, 56)) goto fail;
      tc_fence_after();
#pragma unroll
      for (int j = 0; j < 4; ++j)
        mma_ts(tmem + kTmemO, tmem + kTmemS + slot * 64 + j * 8, desc_at(vd, slot * kVal * kSlab + j * 2048),
               idesc, (i > 0 || j > 0) ? 1u : 0u);
      mma_commit(&sm.pv_done[slot]);
      mma_commit(&sm.val_free[slot]);
    }
    k += T;
  }
  mma_commit(&sm.pv_fin);
  mbar_wait(&sm.pv_fin, 0, 57);
  return;
fail:
  set_abort(sm);
  mma_commit(&sm.pv_fin);
  mbar_wait(&sm.pv_fin, 0, 58);
}

// ---------------------------------------------------------------- softmax
#define MLA_WARP_WAIT(expr) (__all_sync(0xffffffffu, (expr)))

// The fp32 query rows are packed once into bf16 rows [H][d_c + d_r] (q_lat
// then q_rope) in the workspace, so the decode moves half the bytes and can
// load the shared-memory part of a query with TMA.  Eight values per thread.
// The split plan (block 0) and the query packing (the other blocks) in one
// launch; both only read the step's inputs.
__global__ void __launch_bounds__(1024) plan_pack_kernel(const int32_t* __restrict__ seq_lens, int bs, int max_blocks,
                                                         void* ws, DecodeLayout L, const float* __restrict__ q_lat,
                                                         const float* __restrict__ q_rope, long long heads,
                                                         bf16* __restrict__ qpack) {
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0) {
    plan_body(seq_lens, bs, max_blocks, ws, L);
    return;
  }
  constexpr int kPer = kRow / 8;
  for (long long i = (blockIdx.x - 1) * (long long)blockDim.x + threadIdx.x; i < heads * kPer;
       i += (long long)(gridDim.x - 1) * blockDim.x) {
    const long long hrow = i / kPer;
    const int g = (int)(i % kPer);
    const float* src = g < kDc / 8 ? q_lat + hrow * kDc + g * 8 : q_rope + hrow * kDr + (g - kDc / 8) * 8;
    const float4 a = __ldg(reinterpret_cast<const float4*>(src)), b = __ldg(reinterpret_cast<const float4*>(src) + 1);
    *reinterpret_cast<uint4*>(qpack + hrow * kRow + g * 8) =
        make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
  }
}

// Query row v for this CTA: the five shared-memory slabs (the other latent
// half and the rotary part, 128 heads x 64 values each) by TMA, counted on
// q_full; this thread's head row of its own latent half (256 bf16, 512 B)
// from the packed query into TMEM.
__device__ __forceinline__ void load_query(const Params& p, Smem& sm, const CUtensorMap* qmap, int v, int r,
                                           int half, int tid, uint32_t taddr) {
  if (tid == 0) {
    mbar_arrive_expect_tx(&sm.q_full, kEarly * kQSlab);
    for (int i = 0; i < kEarly; ++i) tma_load_2d(sm.qs[i], qmap, early_slab(half, i) * 64, v * kH, &sm.q_full);
  }
  const bf16* qpack = ws_at<bf16>(p.ws, p.L.off_qpack);
  const uint4* src = reinterpret_cast<const uint4*>(qpack + ((long long)v * kH + r) * kRow + 256 * half);
#pragma unroll 1
  for (int b = 0; b < 2; ++b) {  // 2 x 16 loads in flight, 64 columns each
    uint4 w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = __ldg(src + b * 16 + i);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t x[16] = {w[4 * c].x,     w[4 * c].y,     w[4 * c].z,     w[4 * c].w,
                              w[4 * c + 1].x, w[4 * c + 1].y, w[4 * c + 1].z, w[4 * c + 1].w,
                              w[4 * c + 2].x, w[4 * c + 2].y, w[4 * c + 2].z, w[4 * c + 2].w,
                              w[4 * c + 3].x, w[4 * c + 3].y, w[4 * c + 3].z, w[4 * c + 3].w};
      tmem_st16(taddr + kTmemQ + b * 64 + c * 16, x);
    }
  }
}

// The next query row into L2: its five slabs (tensor prefetch, one thread)
// and this thread's TMEM part (four 128-byte lines).
__device__ __forceinline__ void prefetch_query(const Params& p, const CUtensorMap* qmap, int v, int r, int half,
                                               int tid) {
  if (tid == 0)
    for (int i = 0; i < kEarly; ++i) prefetch_l2_2d(qmap, early_slab(half, i) * 64, v * kH);
  const bf16* qpack = ws_at<bf16>(p.ws, p.L.off_qpack);
  const char* src = reinterpret_cast<const char*>(qpack + ((long long)v * kH + r) * kRow + 256 * half);
  for (int i = 0; i < 4; ++i) prefetch_line(src + i * 128);
}

__device__ void softmax_role(Smem& sm, uint32_t tmem, const Params& p, const CUtensorMap* qmap, int seg_begin,
                             int seg_end, int half, int warp, int lane) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const int qw = warp & 3;                                 // TMEM lane quarter
  const int r = qw * 32 + lane;                            // head row == TMEM lane
  const int tid = (warp - 3) * 32 + lane;                  // 0..127
  const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);  // this warp's lane quarter
  float* part_o = ws_at<float>(p.ws, p.L.off_o);
  float* part_lse = ws_at<float>(p.ws, p.L.off_lse);
  if (seg_begin >= seg_end) return;

  load_query(p, sm, qmap, segs[seg_begin].x, r, half, tid, tl);
  tmem_wait_st();
  tc_fence_before();
  mbar_arrive(&sm.q_ready);

  int k = 0;
  for (int si = seg_begin; si < seg_end; ++si) {
    const int4 sg = segs[si];
    const int v = sg.x, b = v / p.n_q, jq = v % p.n_q;
    const int len_v = p.seq_lens[b] - p.n_q + jq + 1;
    const int T = sg.z - sg.y;
    if (si + 1 < seg_end) prefetch_query(p, qmap, segs[si + 1].x, r, half, tid);

    float m_used = -INFINITY, l = 0.f;
    for (int i = 0; i < T; ++i) {
      const int kk = k + i, slot = kk & 1, blk = sg.y + i;
      if (!MLA_WARP_WAIT(mbar_wait(&sm.s_full[slot], ((uint32_t)kk >> 1) & 1, 60))) goto fail;
      tc_fence_after();
      float s[64];
      {
        uint32_t a[32], c2[32];
        tmem_ld32(tl + kTmemS + slot * 64, a);
        tmem_ld32(tl + kTmemS + slot * 64 + 32, c2);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          s[t] = __uint_as_float(a[t]);
          s[32 + t] = __uint_as_float(c2[t]);
        }
      }
      // scale, mask past the row's visible length, row max
      const int valid = max(0, min(kBS, len_v - blk * kBS));
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll
      for (int t = 0; t < 64; ++t) {
        s[t] = t < valid ? s[t] * p.scale_log2 : -INFINITY;
        m8[t & 7] = fmaxf(m8[t & 7], s[t]);
      }
      const float mx =
          fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      bool rescale = false;
      float alpha = 1.f;
      if (i == 0) {
        m_used = mx;
      } else if (mx > m_used + kRescaleLog2) {  // lazy: rescale only when P could grow past 2^8
        alpha = fast_exp2(m_used - mx);
        m_used = mx;
        rescale = true;
      }
      const float mbase = m_used == -INFINITY ? 0.f : m_used;  // a fully masked page gives P = 0, not NaN
      uint32_t pk[32];
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const float p0 = fast_exp2(s[2 * t] - mbase), p1 = fast_exp2(s[2 * t + 1] - mbase);
        ps[t & 3] += p0 + p1;
        pk[t] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));

      // tcgen05.ld / st are warp-collective: the warp rescales when any row needs it.
      if (__any_sync(0xffffffffu, rescale)) {
        // O must hold every earlier page before it is scaled: wait for P V of page kk - 1.
        if (!MLA_WARP_WAIT(mbar_wait(&sm.pv_done[slot ^ 1], ((uint32_t)(kk - 1) >> 1) & 1, 61))) goto fail;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          const uint32_t a = tl + kTmemO + c * 32;
          tmem_ld32(a, o);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
          tmem_st32(a, o);
        }
      }
      if (valid < kBS) {
        // Rows past the visible length hold whatever the pool holds (maybe
        // NaN); P is 0 there, but 0 x NaN is NaN, so clear them in the value slabs.
        const int nrow = kBS - valid, per_slab = nrow * 8;
        for (int c = tid; c < kVal * per_slab; c += 32 * kSoftmaxWarps) {
          const int e = c / per_slab, rem = c % per_slab;
          *reinterpret_cast<uint4*>(sm.val[slot][e] + (valid + rem / 8) * 128 + (rem % 8) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      tmem_st32(tl + kTmemS + slot * 64, pk);  // P over the page's own scores
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_ready[slot]);
    }
    // The scores of this segment are all done: the next query can replace this one.
    if (si + 1 < seg_end) {
      load_query(p, sm, qmap, segs[si + 1].x, r, half, tid, tl);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.q_ready);
    }
    {
      // epilogue of the segment: O half / l and the log2-sum-exp
      const int kl = k + T - 1;
      if (!MLA_WARP_WAIT(mbar_wait(&sm.pv_done[kl & 1], ((uint32_t)kl >> 1) & 1, 62))) goto fail;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      // head-minor partial output: the warp's 32 heads of one column are one 128-byte line
      float* out = part_o + ((long long)si * kDc + half * 256) * kH + r;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        tmem_ld32(tl + kTmemO + c * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) out[(long long)(c * 32 + t) * kH] = __uint_as_float(o[t]) * inv;
      }
      tc_fence_before();
      if (half == 0) part_lse[(long long)si * kH + r] = l > 0.f ? m_used + log2f(l) : -INFINITY;
    }
    k += T;
  }
  return;
fail:
  set_abort(sm);
}

// ---------------------------------------------------------------- kernel
__global__ void __launch_bounds__(kThreads, 1) decode_tc3_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                  const __grid_constant__ CUtensorMap qmap,
                                                                  const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int worker = blockIdx.x >> 1, half = blockIdx.x & 1;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.early_full[b], 1);
      mbar_init(&sm.val_full[b], 1);
      mbar_init(&sm.early_free[b], 1);
      mbar_init(&sm.val_free[b], 1);
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.p_ready[b], 32 * kSoftmaxWarps);
      mbar_init(&sm.pv_done[b], 1);
    }
    mbar_init(&sm.q_ready, 32 * kSoftmaxWarps);
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.s_fin, 1);
    mbar_init(&sm.pv_fin, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap);
    prefetch_tensormap(&qmap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();  // the plan, the packed query and the appended rows come from the kernels before
  pdl_trigger();

  int seg_begin = 0, seg_end = 0;
  if (worker < p.L.workers) {
    const int* wfirst = ws_at<int>(p.ws, p.L.off_worker_first);
    seg_begin = wfirst[worker];
    seg_end = wfirst[worker + 1];
  }

  // The single-thread roles keep their warp's other lanes parked at a warp
  // barrier (not at the CTA barrier below) while lane 0 works.
  if (warp == 0) {
    if (lane == 0) producer(sm, &tmap, p, seg_begin, seg_end, half);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) score_issuer(sm, tmem, p, seg_begin, seg_end);
    __syncwarp();
  } else if (warp == 2) {
    if (lane == 0) pv_issuer(sm, tmem, p, seg_begin, seg_end);
    __syncwarp();
  } else {
    softmax_role(sm, tmem, p, &qmap, seg_begin, seg_end, half, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

#undef MLA_WARP_WAIT

}  // namespace tcdec3
}  // namespace mla
