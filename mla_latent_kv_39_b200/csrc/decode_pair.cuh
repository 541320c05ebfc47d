// Latent-space split-KV decode on pairs of SMs (tcgen05 .cta_group::2).
//
// "MLA · latent KV, decoupled RoPE và matrix absorption" (openarchlab),
// section 1 "Định nghĩa" and section 2 "Luồng": with W_UK absorbed into the
// query and W_UV into the output side, for every head h of query row v
//   s_t = q_lat[h] . c_t + q_R[h] . k_R,t          (t over the visible rows)
//   o_lat[h] = sum_t softmax(scale * s)_t c_t        (the latent output)
// The split-KV plan (decode_plan.cuh) hands every worker one contiguous run
// of pages (one or more query rows, "segments"); per segment the worker
// writes the normalised partial output (bf16, [segment][head][d]) and its
// log2-sum-exp.
//
// A worker is a cluster of two CTAs on two SMs.  CTA r owns heads
// [64 r, 64 r + 64): its TMEM holds those heads' scores and their whole
// 512-wide latent output.  The pages are walked two at a time (a 128-token
// tile).  The scores of a tile are one pair MMA per 16-value K step, M = 128
// heads (A split by heads), N = 128 tokens (B split by pages: CTA r holds
// page r of the tile, all 576 values), so every page is read from memory
// once and every score is computed once.  P V is a pair MMA per 16 tokens
// and 128-column latent chunk m, N split by columns: CTA r supplies columns
// 128 m + 64 r + (0..63), which for its own page is its score slab 2 m + r,
// kept in place, and for the other page is that page's slab 2 m + r,
// fetched into the slot of the other CTA's matching slab once the scores
// have read it (an L2 hit: the other CTA has just loaded that page).  The
// rows of D that a pair MMA leaves in one CTA's TMEM sit in 128 lanes x N/2
// columns: lane l holds head 64 r + (l mod 64), lanes 0..63 the first half
// of the N columns and lanes 64..127 the second.
//
// Warp roles (224 threads per CTA): warp 0 issues the score-side TMA loads
// and warp 6 the value-side ones (both CTAs, counted on the leader's
// barriers); warp 1 of the leader issues every MMA of the pair; warps 2..5
// run the online softmax, one TMEM lane per thread (a head and one page of
// the tile), and write the segment's partial output.  Per tile the tensor
// pipe runs the scores, then (once the softmax has written P) P V, so the
// previous tile's P V is over when the next scores arrive.
//
// TMEM (512 columns): [0,64) the score tile, [64,320) the latent output
// (four 64-column chunks), [320,512) the query's latent columns 0..383 (A of
// the first 24 score K steps).
//
// Shared memory: the query's last 3 K slabs (64 heads x 64 values, 128-byte
// swizzle, K-major), P (2 pages x 64 heads x 64 tokens) and a ring of 8 KiB
// slots for page slabs (and, in split-query mode, the low query slabs).
//
// The last page of a row may be partial: it is loaded with its row
// coordinate shifted down by the missing rows, so the rows past the visible
// length arrive as zeros (out-of-range fill) at the top of the tile and the
// pool's contents there (maybe NaN) are never read.  A tile with only one
// page skips the second page's loads and its P V steps.
//
// Every wait gives up after a time limit, records MLA_ERR_TIMEOUT and makes
// the roles wind down.
#pragma once

#include "decode_plan.cuh"
#include "sm100.cuh"

namespace mla {
namespace pairdec {

using namespace sm100;

constexpr int kH = 128, kHalfH = 64, kDc = 512, kDr = 64, kBS = 64, kRow = kDc + kDr;
constexpr int kSlabs = kRow / 64;  // 9 K slabs of 64 values
constexpr int kTmemQSlabs = 6;     // query K slabs held in TMEM (latent columns 0..383)
constexpr int kSmemQSlabs = kSlabs - kTmemQSlabs;
constexpr int kVSlabs = kDc / 64;  // 8 slabs hold latent (value) columns, the ninth the rotary key
constexpr int kSlab = 64 * 128;    // 64 rows x 64 bf16, 128-byte swizzle
// Ring of 8 KiB slots (build-time tunable; the default fills the 227 KiB of
// shared memory beside the query and P buffers).
#ifndef MLA_PAIR_RING
#define MLA_PAIR_RING 22
#endif
// How far (in K slabs) the score-side loads of a tile may run ahead of the
// previous tile's score MMAs.  The SM's TMA engine serves loads in issue
// order, so a whole tile of score slabs issued early would queue the
// previous tile's value reloads (needed sooner, by its P V) behind them.
#ifndef MLA_PAIR_AHEAD
#define MLA_PAIR_AHEAD 3
#endif
constexpr int kRing = MLA_PAIR_RING, kAhead = MLA_PAIR_AHEAD;
constexpr int kTmemS = 0, kTmemO = 64, kTmemQ = 320, kTmemCols = 512;
constexpr int kSoftmaxWarps = 4;
constexpr int kSoftmaxWarp0 = 2;                    // warps 2..5
constexpr int kVcWarp = kSoftmaxWarp0 + kSoftmaxWarps;
constexpr int kThreads = 32 * (kVcWarp + 1);
constexpr float kRescaleLog2 = 8.f;
constexpr uint16_t kBoth = 3;  // multicast mask: both CTAs of the pair

struct Smem {
  uint8_t q[kSmemQSlabs][kSlab];  // query K slabs 6..8; first member: 1024-byte aligned
  uint8_t p[2][kSlab];            // P of the tile: [page of the tile] 64 heads x 64 tokens
  uint8_t ring[kRing][kSlab];     // page slabs (and low query slabs)
  uint64_t full[kRing], qkd[kRing], vfull[kRing], empty[kRing];
  uint64_t q_full, q_empty, qt_full;
  uint64_t s_full, s_free, p_full, pv_done;
  uint64_t o_free, fin, xbar[2], lbar;
  float xm[2][128];  // tile max of each TMEM lane (exchanged between lanes l and l ^ 64)
  float xl[128];     // row sums at the end of a segment
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory over the 227 KiB per-block limit");

struct Params {
  const bf16* q;  // packed query rows [rows][H][576] (the TMEM part is read from here)
  const int32_t* block_table;
  const int32_t* seq_lens;
  int max_blocks, num_blocks, n_q, split;
  float scale_log2;
  unsigned long long wait_ns;
  void* ws;
  DecodeLayout L;
};

__device__ __forceinline__ void set_abort(Smem& sm) { *(volatile int*)&sm.abort_flag = 1; }
__device__ __forceinline__ bool aborted(Smem& sm) { return *(volatile int*)&sm.abort_flag != 0; }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The same barrier in the leader CTA (rank 0), as a shared::cluster address.
__device__ __forceinline__ uint32_t leader(const uint64_t* bar) { return mapa(smem_u32(bar), 0); }

__device__ __forceinline__ uint64_t kmajor_desc(const void* p, uint32_t byte_off) {
  return smem_desc(smem_u32(p) + byte_off, 16, 1024, kSwizzle128B);
}

// Descriptors differ only in the start address (bits 0-13, 16-byte units).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t byte_offset) { return d + (byte_offset >> 4); }

// ---------------------------------------------------------------- tiles
// Walks the worker's tiles in order: segment, first page of the tile.
struct Tiles {
  const int4* segs;
  int si, seg_end, pg, nseg;  // nseg: segments started so far (this one included)
  __device__ Tiles(const int4* s, int b, int e) : segs(s), si(b), seg_end(e), pg(b < e ? s[b].y : 0), nseg(1) {}
  __device__ bool valid() const { return si < seg_end; }
  __device__ int4 seg() const { return segs[si]; }
  __device__ bool first() const { return pg == segs[si].y; }
  __device__ bool last() const { return pg + 2 >= segs[si].z; }
  __device__ bool has_b() const { return pg + 1 < segs[si].z; }
  __device__ void next() {
    pg += 2;
    if (pg >= segs[si].z && ++si < seg_end) {
      pg = segs[si].y;
      ++nseg;
    }
  }
};

// Visible rows of query row v: its sequence's rows up to and including its own.
__device__ __forceinline__ int visible_len(const Params& p, int v) {
  const int b = v / p.n_q, j = v % p.n_q;
  return p.seq_lens[b] - p.n_q + j + 1;
}

__device__ __forceinline__ int page_valid(int len_v, int blk) { return max(0, min(kBS, len_v - blk * kBS)); }

__device__ __forceinline__ int phys_block(const Params& p, int v, int blk, bool report_err) {
  const int b = v / p.n_q;
  int phys = p.block_table[(long long)b * p.max_blocks + blk];
  if (phys < 0 || phys >= p.num_blocks) {
    if (report_err) report(MLA_ERR_BOUNDS, 5, b, phys);
    phys = 0;  // keep the pipeline moving; the error word marks the result invalid
  }
  return phys;
}

// ---------------------------------------------------------------- ring items
// Per tile every role walks the same item sequence: for K slab e = 0..8 a
// page item (this CTA's page slab e), followed in split-query mode by a low
// query item (the slab e of the query's bf16 remainder).  Item n lives in
// ring slot n mod kRing.  A page item with e < 8 is kept until the tile's
// P V: one CTA of the pair keeps its own slab, the other replaces its slab,
// once the scores have read it, by the matching value slab of the other page
// (see the header comment); the rotary slab and low query items are freed
// right after the scores.
struct Items {
  int per_tile;
  __device__ explicit Items(int split) : per_tile(split ? 2 * kSlabs : kSlabs) {}
  __device__ uint32_t page(int tile, int e) const { return (uint32_t)(tile * per_tile + e * (per_tile / kSlabs)); }
};

// Per-slot use counters of the barriers that not every item uses.
struct SlotUses {
  uint8_t n[kRing];
  __device__ SlotUses() {
    for (int i = 0; i < kRing; ++i) n[i] = 0;
  }
  __device__ uint32_t next(int slot) { return n[slot]++ & 1u; }
};

// Which CTA of the pair fetches the other page's half for value slab e, and
// which slab of which page of the tile that is: for even e = 2m CTA 1 needs
// page 0's slab 2m + 1; for odd e = 2m + 1 CTA 0 needs page 1's slab 2m.
__device__ __forceinline__ uint32_t reloader(int e) { return (e & 1) ? 0u : 1u; }
__device__ __forceinline__ int reload_page(int e) { return (e & 1) ? 1 : 0; }
__device__ __forceinline__ int reload_slab(int e) { return (e & 1) ? e - 1 : e + 1; }

// ---------------------------------------------------------------- TMA producers
// Score-side loads (warp 0): the segment's query slabs held in shared
// memory, then per tile the 9 slabs of this CTA's page (and the low query
// slabs), each into the next ring slot once its previous use is over.
__device__ void producer_k(Smem& sm, const CUtensorMap* pool, const CUtensorMap* qmap, const CUtensorMap* qlomap,
                           const Params& p, int seg_begin, int seg_end, uint32_t rank) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const bool lead = rank == 0;
  const Items items(p.split);
  SlotUses qkd_use;
  uint32_t n = 0;  // items issued
  int nq = 0;      // query loads issued
  int ti = 0;
  for (Tiles t(segs, seg_begin, seg_end); t.valid() && !aborted(sm); t.next(), ++ti) {
    // phases of the previous tile's "scores have read value slab e" barriers
    uint32_t prev_qkd[kVSlabs];
    if (ti >= 1)
      for (int e = 0; e < kVSlabs; ++e) prev_qkd[e] = qkd_use.next((int)(items.page(ti - 1, e) % kRing));
    const int v = t.seg().x;
    if (t.first()) {
      if (nq >= 1 && !mbar_wait(&sm.q_empty, (nq - 1) & 1, 70, p.wait_ns)) goto fail;
      if (lead) mbar_arrive_expect_tx(&sm.q_full, 2 * kSmemQSlabs * kSlab);
      for (int e = kTmemQSlabs; e < kSlabs; ++e)
        tma_load_2d_pair(sm.q[e - kTmemQSlabs], qmap, 64 * e, v * kH + kHalfH * (int)rank, leader(&sm.q_full));
      ++nq;
    }
    const bool has = rank == 0 || t.has_b();
    const int blk = t.pg + (int)rank;
    const int phys = has ? phys_block(p, v, blk, true) : 0;
    const int y = has ? page_valid(visible_len(p, v), blk) - kBS : 0;
    const uint32_t page_bytes = (t.has_b() ? 2 : 1) * kSlab;
    for (int e = 0; e < kSlabs; ++e) {
      if (ti >= 1) {  // pace: the previous tile's scores have read slab e + kAhead
        const int ea = e + kAhead;
        const bool ok = ea < kVSlabs
                            ? mbar_wait(&sm.qkd[items.page(ti - 1, ea) % kRing], prev_qkd[ea], 74, p.wait_ns)
                            : mbar_wait(&sm.s_full, (ti - 1) & 1, 75, p.wait_ns);
        if (!ok) goto fail;
      }
      for (int lo = 0; lo <= p.split; ++lo, ++n) {
        const int slot = (int)(n % kRing);
        const uint32_t use = n / kRing;
        if (use >= 1 && !mbar_wait(&sm.empty[slot], (use - 1) & 1, 71, p.wait_ns)) goto fail;
        if (lo == 0) {
          if (lead) mbar_arrive_expect_tx(&sm.full[slot], page_bytes);
          if (has) tma_load_3d_pair(sm.ring[slot], pool, 64 * e, y, phys, leader(&sm.full[slot]));
        } else {  // the low part of the query for the same K slab
          if (lead) mbar_arrive_expect_tx(&sm.full[slot], 2 * kSlab);
          tma_load_2d_pair(sm.ring[slot], qlomap, 64 * e, v * kH + kHalfH * (int)rank, leader(&sm.full[slot]));
        }
      }
    }
  }
  return;
fail:
  set_abort(sm);
}

// Value-side loads (warp 6): once the scores have read value slab e of a
// tile, the CTA that does not keep it fetches the other page's matching slab
// into the same slot (it is in L2: the other CTA loaded that page for its
// scores); the leader counts the bytes.
__device__ void producer_v(Smem& sm, const CUtensorMap* pool, const Params& p, int seg_begin, int seg_end,
                           uint32_t rank) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const bool lead = rank == 0;
  const Items items(p.split);
  SlotUses qkd_use;
  int ti = 0;
  for (Tiles t(segs, seg_begin, seg_end); t.valid() && !aborted(sm); t.next(), ++ti) {
    const int v = t.seg().x, len_v = visible_len(p, v);
    for (int e = 0; e < kVSlabs; ++e) {
      const int slot = (int)(items.page(ti, e) % kRing);
      if (!mbar_wait(&sm.qkd[slot], qkd_use.next(slot), 73, p.wait_ns)) goto fail;
      const int pgi = reload_page(e);
      const bool exists = pgi == 0 || t.has_b();
      if (lead) mbar_arrive_expect_tx(&sm.vfull[slot], exists ? kSlab : 0);
      if (exists && rank == reloader(e)) {
        const int blk = t.pg + pgi;
        tma_load_3d_pair(sm.ring[slot], pool, 64 * reload_slab(e), page_valid(len_v, blk) - kBS,
                         phys_block(p, v, blk, false), leader(&sm.vfull[slot]));
      }
    }
  }
  return;
fail:
  set_abort(sm);
}

// ---------------------------------------------------------------- MMA issuer (leader CTA)
// Per tile: the score MMAs over the 9 K slabs, then (after the softmax has
// written P) P V, one 128-column latent chunk m at a time: its page-0 half
// from value slab item 2m, its page-1 half from item 2m + 1.
__device__ void mma_issuer(Smem& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, 0, 1);
  const uint64_t wns = p.wait_ns;
  const Items items(p.split);
  SlotUses vfull_use;
  int ti = 0;
  for (Tiles t(segs, seg_begin, seg_end); t.valid(); t.next(), ++ti) {
    // ---- scores
    if (t.first() && (!mbar_wait(&sm.q_full, (t.nseg - 1) & 1, 80, wns) ||
                      !mbar_wait(&sm.qt_full, (t.nseg - 1) & 1, 79, wns)))
      goto fail;
    if (ti >= 1 && !mbar_wait(&sm.s_free, (ti - 1) & 1, 81, wns)) goto fail;
    tc_fence_after();
    for (int e = 0; e < kSlabs; ++e) {
      const uint32_t n = items.page(ti, e);
      const int slot = (int)(n % kRing);
      if (!mbar_wait(&sm.full[slot], (n / kRing) & 1, 82, wns)) goto fail;
      int lo_slot = 0;
      if (p.split) {
        lo_slot = (int)((n + 1) % kRing);
        if (!mbar_wait(&sm.full[lo_slot], ((n + 1) / kRing) & 1, 83, wns)) goto fail;
      }
      tc_fence_after();
      const uint32_t d = tmem + kTmemS;
      if (e < kTmemQSlabs) {  // A (query) from TMEM: 8 columns of bf16 pairs per 16-value K step
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_ts_pair(d, tmem + kTmemQ + 32 * e + 8 * j, kmajor_desc(sm.ring[slot], 32 * j), idesc_s,
                      (e | j) ? 1u : 0u);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_ss_pair(d, kmajor_desc(sm.q[e - kTmemQSlabs], 32 * j), kmajor_desc(sm.ring[slot], 32 * j), idesc_s, 1u);
      }
      if (p.split) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_ss_pair(d, kmajor_desc(sm.ring[lo_slot], 32 * j), kmajor_desc(sm.ring[slot], 32 * j), idesc_s, 1u);
        mma_commit_pair(&sm.empty[lo_slot], kBoth);
      }
      mma_commit_pair(e < kVSlabs ? &sm.qkd[slot] : &sm.empty[slot], kBoth);
    }
    mma_commit_pair(&sm.s_full, kBoth);
    if (t.last()) mma_commit_pair(&sm.q_empty, kBoth);

    // ---- P V
    if (t.first() && t.nseg >= 2 && !mbar_wait(&sm.o_free, (t.nseg - 2) & 1, 84, wns)) goto fail;
    if (!mbar_wait(&sm.p_full, ti & 1, 85, wns)) goto fail;
    tc_fence_after();
    for (int e = 0; e < kVSlabs; ++e) {
      const int m = e >> 1, pgi = e & 1;
      const int slot = (int)(items.page(ti, e) % kRing);
      if (!mbar_wait(&sm.vfull[slot], vfull_use.next(slot), 86, wns)) goto fail;
      if (pgi == 0 || t.has_b()) {
        tc_fence_after();
        // value slab as an MN-major B operand: 64 latent columns, 8-token
        // groups 1 KiB apart (SBO), 16 tokens per K step
        const uint64_t vd = smem_desc(smem_u32(sm.ring[slot]), kSlab, 1024, kSwizzle128B);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss_pair(tmem + kTmemO + 64 * m, kmajor_desc(sm.p[pgi], 32 * kk), desc_add(vd, 2048 * kk), idesc_o,
                      (t.first() && pgi == 0 && kk == 0) ? 0u : 1u);
      }
      mma_commit_pair(&sm.empty[slot], kBoth);
    }
    mma_commit_pair(&sm.pv_done, kBoth);
  }
  mma_commit_pair(&sm.fin, 1);
  mbar_wait(&sm.fin, 0, 87, wns);
  return;
fail:
  set_abort(sm);
  mma_commit_pair(&sm.fin, 1);
  mbar_wait(&sm.fin, 0, 88, wns);
}

// ---------------------------------------------------------------- softmax
#define MLA_WARP_WAIT(expr) (__all_sync(0xffffffffu, (expr)))

// The query's latent columns 0..383 of this lane's head into TMEM (the A
// operand of the first 24 score K steps).  A pair MMA with A in TMEM reads
// each CTA's 64 rows from lanes 0..63 and again from lanes 64..127, so lanes
// l and l ^ 64 both hold head 64 r + (l mod 64).  Then the leader is told.
__device__ __forceinline__ void load_query_tmem(Smem& sm, const Params& p, int v, int head, uint32_t tl, int lane) {
  const uint4* src = reinterpret_cast<const uint4*>(p.q + ((long long)v * kH + head) * kRow);
#pragma unroll 1
  for (int b = 0; b < kTmemQSlabs / 2; ++b) {  // 16 loads in flight per round, 64 columns each
    uint4 w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = __ldg(src + b * 16 + i);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t x[16] = {w[4 * c].x,     w[4 * c].y,     w[4 * c].z,     w[4 * c].w,
                              w[4 * c + 1].x, w[4 * c + 1].y, w[4 * c + 1].z, w[4 * c + 1].w,
                              w[4 * c + 2].x, w[4 * c + 2].y, w[4 * c + 2].z, w[4 * c + 2].w,
                              w[4 * c + 3].x, w[4 * c + 3].y, w[4 * c + 3].z, w[4 * c + 3].w};
      tmem_st16(tl + kTmemQ + b * 64 + c * 16, x);
    }
  }
  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive_remote(leader(&sm.qt_full));
}

__device__ void softmax_role(Smem& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end, uint32_t rank,
                             int warp, int lane) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const int qw = warp & 3;                                 // TMEM lane quarter
  const int l = qw * 32 + lane;                            // TMEM lane
  const int half = l >> 6;                                 // page of the tile / latent half of O
  const int hl = l & 63, head = kHalfH * (int)rank + hl;   // head of this lane
  const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);  // this warp's lane quarter
  const uint64_t wns = p.wait_ns;
  bf16* part_o = ws_at<bf16>(p.ws, p.L.off_o);
  float* part_lse = ws_at<float>(p.ws, p.L.off_lse);

  float m_used = -INFINITY, lsum = 0.f;
  int nseg_done = 0;
  Tiles t(segs, seg_begin, seg_end);
  if (t.valid()) load_query_tmem(sm, p, t.seg().x, head, tl, lane);
  for (int i = 0; t.valid(); ++i, t.next()) {
    const int4 sg = t.seg();
    const int v = sg.x, len_v = visible_len(p, v);
    const bool first = t.first(), last = t.last();
    if (first) {
      m_used = -INFINITY;
      lsum = 0.f;
    }
    if (!MLA_WARP_WAIT(mbar_wait(&sm.s_full, i & 1, 90, wns))) goto fail;
    tc_fence_after();
    float s[64];
    {
      uint32_t a[32], b[32];
      tmem_ld32(tl + kTmemS, a);
      tmem_ld32(tl + kTmemS + 32, b);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        s[c] = __uint_as_float(a[c]);
        s[32 + c] = __uint_as_float(b[c]);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_remote(leader(&sm.s_free));

    // this lane's page: rows past the visible length sit at the top of the tile
    const int blk = t.pg + half;
    const int shift = kBS - ((half == 0 || t.has_b()) ? page_valid(len_v, blk) : 0);
    float m8[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) m8[c] = -INFINITY;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
      s[c] = c >= shift ? s[c] * p.scale_log2 : -INFINITY;
      m8[c & 7] = fmaxf(m8[c & 7], s[c]);
    }
    const float m_loc =
        fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
    sm.xm[i & 1][l] = m_loc;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.xbar[i & 1]);
    if (!MLA_WARP_WAIT(mbar_wait(&sm.xbar[i & 1], (i >> 1) & 1, 91, wns))) goto fail;
    const float m_tile = fmaxf(m_loc, sm.xm[i & 1][l ^ 64]);

    bool rescale = false;
    float alpha = 1.f;
    if (first) {
      m_used = m_tile;
    } else if (m_tile > m_used + kRescaleLog2) {  // lazy: rescale only when P could grow past 2^8
      alpha = fast_exp2(m_used - m_tile);
      m_used = m_tile;
      rescale = true;
    }
    const float mbase = m_used == -INFINITY ? 0.f : m_used;
    uint32_t pk[32];
    float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const float p0 = fast_exp2(s[2 * c] - mbase), p1 = fast_exp2(s[2 * c + 1] - mbase);
      ps[c & 3] += p0 + p1;
      pk[c] = pack_bf16x2(p0, p1);
    }
    lsum = lsum * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));

    // O holds every earlier tile (their P V ran before this tile's scores on
    // the in-order tensor pipe).  tcgen05.ld / st are warp-collective: the
    // warp rescales when any lane needs it.
    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        const uint32_t a = tl + kTmemO + c * 32;
        tmem_ld32(a, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
        tmem_st32(a, o);
      }
      tmem_wait_st();
    }
    {
      // row hl of this page's P slab, K-major with the 128-byte swizzle (the
      // previous tile's P V is over: this tile's scores ran after it)
      uint8_t* row = sm.p[half] + hl * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(row + ((c ^ (hl & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_remote(leader(&sm.p_full));

    // The scores of this segment are all done (s_full of its last tile): the
    // next segment's query can replace this one in TMEM, before the epilogue,
    // which waits for this tile's P V (queued before the next segment's scores).
    if (last && t.si + 1 < seg_end) load_query_tmem(sm, p, segs[t.si + 1].x, head, tl, lane);

    if (last) {
      // epilogue of the segment: O / l and the log2-sum-exp
      sm.xl[l] = lsum;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.lbar);
      if (!MLA_WARP_WAIT(mbar_wait(&sm.lbar, nseg_done & 1, 94, wns))) goto fail;
      const float ltot = lsum + sm.xl[l ^ 64];
      if (!MLA_WARP_WAIT(mbar_wait(&sm.pv_done, i & 1, 95, wns))) goto fail;
      tc_fence_after();
      const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
      const int si = t.si;
      // partial output [segment][head][d] in bf16: chunk m of O holds latent
      // columns 128 m + 64 half + (0..63) in this lane
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        tmem_ld32(tl + kTmemO + c * 32, o);
        tmem_wait_ld();
        const int d0 = 128 * (c >> 1) + 64 * half + 32 * (c & 1);
        uint4* out = reinterpret_cast<uint4*>(part_o + ((long long)si * kH + head) * kDc + d0);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float* f = reinterpret_cast<const float*>(o) + 8 * k;
          out[k] = make_uint4(pack_bf16x2(f[0] * inv, f[1] * inv), pack_bf16x2(f[2] * inv, f[3] * inv),
                              pack_bf16x2(f[4] * inv, f[5] * inv), pack_bf16x2(f[6] * inv, f[7] * inv));
        }
      }
      if (half == 0) part_lse[(long long)si * kH + head] = ltot > 0.f ? m_used + log2f(ltot) : -INFINITY;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(leader(&sm.o_free));
      ++nseg_done;
    }
  }
  return;
fail:
  set_abort(sm);
}

#undef MLA_WARP_WAIT

// ---------------------------------------------------------------- plan + query pack
// The split plan (block 0) and the query packing (the other blocks) in one
// launch.  The fp32 query rows are packed into bf16 rows [H][d_c + d_r]
// (q_lat then q_rope) so the decode loads them with TMA; in split-query mode
// a second copy holds the bf16 remainder q - bf16(q).
__global__ void __launch_bounds__(1024) pair_plan_pack_kernel(const int32_t* __restrict__ seq_lens, int bs,
                                                              int max_blocks, void* ws, DecodeLayout L,
                                                              const float* __restrict__ q_lat,
                                                              const float* __restrict__ q_rope, long long heads,
                                                              bf16* __restrict__ qpack, bf16* __restrict__ qlo) {
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
    const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      hi[k] = pack_bf16x2(x[2 * k], x[2 * k + 1]);
      const float h0 = __uint_as_float(hi[k] << 16), h1 = __uint_as_float(hi[k] & 0xFFFF0000u);
      lo[k] = pack_bf16x2(x[2 * k] - h0, x[2 * k + 1] - h1);
    }
    *reinterpret_cast<uint4*>(qpack + hrow * kRow + g * 8) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    if (qlo != nullptr)
      *reinterpret_cast<uint4*>(qlo + hrow * kRow + g * 8) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// ---------------------------------------------------------------- kernel
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_pair_kernel(const __grid_constant__ CUtensorMap pool, const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap qlomap, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int worker = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.qkd[s], 1);
      mbar_init(&sm.vfull[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, 2 * kSoftmaxWarps);
    mbar_init(&sm.p_full, 2 * kSoftmaxWarps);
    mbar_init(&sm.pv_done, 1);
    for (int b = 0; b < 2; ++b) mbar_init(&sm.xbar[b], kSoftmaxWarps);
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    mbar_init(&sm.qt_full, 2 * kSoftmaxWarps);
    mbar_init(&sm.o_free, 2 * kSoftmaxWarps);
    mbar_init(&sm.fin, 1);
    mbar_init(&sm.lbar, kSoftmaxWarps);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&pool);
    prefetch_tensormap(&qmap);
    if (p.split) prefetch_tensormap(&qlomap);
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive or load
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
    if (lane == 0) producer_k(sm, &pool, &qmap, &qlomap, p, seg_begin, seg_end, rank);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) mma_issuer(sm, tmem, p, seg_begin, seg_end);
    __syncwarp();
  } else if (warp == kVcWarp) {
    if (lane == 0) producer_v(sm, &pool, p, seg_begin, seg_end, rank);
    __syncwarp();
  } else {
    softmax_role(sm, tmem, p, seg_begin, seg_end, rank, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair's MMAs and remote arrives are over before TMEM and shared memory go away
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ================================================================ host side
inline bool supports(const mla_config* c) {
  return c->dtype == MLA_BF16 && c->n_heads == kH && c->d_c == kDc && c->d_r == kDr && c->block_size == kBS;
}

// Bytes of packed query the decode keeps in its workspace per query row
// (the bf16 query, and its bf16 remainder in split-query mode).
inline size_t qpack_row_bytes(const mla_config* c) {
  const bool split = (c->flags & MLA_FLAG_SPLIT_QUERY) != 0;
  return (size_t)kH * kRow * sizeof(bf16) * (split ? 2 : 1);
}

// The pool as a 3-D bf16 tensor [num_blocks][64 rows][576 values] (row
// stride 1152 B, page stride 73,728 B), read in boxes of 64 values x 64 rows
// of one page with the 128-byte swizzle; rows outside the page read as zero.
inline mla_status pool_map(const mla_cache* k, CUtensorMap* map) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return MLA_ERR_CUDA;
  const cuuint64_t dims[3] = {(cuuint64_t)kRow, (cuuint64_t)kBS, (cuuint64_t)k->num_blocks};
  const cuuint64_t strides[2] = {(cuuint64_t)kRow * 2, (cuuint64_t)kRow * 2 * kBS};
  const cuuint32_t box[3] = {64, (cuuint32_t)kBS, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k->pool, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// A packed query (bf16 [rows * 128 heads, 576]) read in boxes of 64 values x
// 64 heads: one box is one shared-memory query slab of one CTA.
inline mla_status query_map(const void* q, long long rows, CUtensorMap* map) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return MLA_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)kRow, (cuuint64_t)rows * kH};
  const cuuint64_t strides[1] = {(cuuint64_t)kRow * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kHalfH};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

inline mla_status set_smem_once(const void* fn, size_t bytes, std::atomic<uint64_t>& done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done_mask.load(std::memory_order_acquire) & bit)) return MLA_OK;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (bit) done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return MLA_OK;
}

// Plan + query pack, then the pair decode (two chained launches).  With
// `q_packed` (the query already in the packed bf16 layout, from
// mla_absorb_q_packed) the first launch only computes the plan.
inline mla_status launch(const mla_config* c, const float* q_lat, const float* q_rope, const bf16* q_packed, int n_q,
                         const mla_cache* k, const int32_t* seq_lens, void* ws, const DecodeLayout& L, float scale,
                         unsigned long long wait_ns, cudaStream_t s) {
  const bool split = (c->flags & MLA_FLAG_SPLIT_QUERY) != 0;
  const long long rows = (long long)L.batch * L.n_q;
  bf16* qpack = q_packed ? const_cast<bf16*>(q_packed) : reinterpret_cast<bf16*>(static_cast<char*>(ws) + L.off_qpack);
  bf16* qlo = split ? qpack + rows * kH * kRow : nullptr;
  CUtensorMap pmap, qmap, qlomap;
  mla_status st = pool_map(k, &pmap);
  if (st == MLA_OK) st = query_map(qpack, rows, &qmap);
  if (st == MLA_OK) st = query_map(split ? qlo : qpack, rows, &qlomap);
  if (st != MLA_OK) return st;

  static std::atomic<uint64_t> plan_attr{0}, plan_only_attr{0}, dec_attr{0};
  const size_t plan_smem = sizeof(int) * ((size_t)rows + 1);
  if (set_smem_once((const void*)decode_pair_kernel, kSmemBytes, dec_attr) != MLA_OK) return MLA_ERR_CUDA;
  if (q_packed) {
    if (plan_smem > 48 * 1024 && set_smem_once((const void*)decode_plan_kernel, plan_smem, plan_only_attr) != MLA_OK)
      return MLA_ERR_CUDA;
    if (launch_chained(decode_plan_kernel, dim3(1), dim3(1024), plan_smem, s, seq_lens, c->block_size,
                       k->max_blocks_per_seq, ws, L) != cudaSuccess)
      return MLA_ERR_CUDA;
  } else {
    if (plan_smem > 48 * 1024 && set_smem_once((const void*)pair_plan_pack_kernel, plan_smem, plan_attr) != MLA_OK)
      return MLA_ERR_CUDA;
    const long long groups = rows * kH * (kRow / 8);
    const int qblocks = (int)std::min<long long>((groups + 1023) / 1024, 4096);
    if (launch_chained(pair_plan_pack_kernel, dim3(1 + qblocks), dim3(1024), plan_smem, s, seq_lens, c->block_size,
                       k->max_blocks_per_seq, ws, L, q_lat, q_rope, rows * kH, qpack, qlo) != cudaSuccess)
      return MLA_ERR_CUDA;
  }
  const Params p{qpack, k->block_table, seq_lens, k->max_blocks_per_seq, k->num_blocks, n_q, split ? 1 : 0,
                 scale * 1.4426950408889634f, wait_ns, ws, L};
  return launch_chained(decode_pair_kernel, dim3(2 * L.workers), dim3(kThreads), kSmemBytes, s, pmap, qmap, qlomap,
                        p) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

}  // namespace pairdec
}  // namespace mla
