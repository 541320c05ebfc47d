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
// tile; CTA r loads page r of the tile).
//
// Scores: one pair MMA per 16-value K step, M = 128 heads (A split by
// heads), N = 128 tokens (B split by pages), so every page is read from
// memory once and every score is computed once.
//
// P V: one pair MMA per 16 tokens of a page and 256-column latent block j,
// N = 256 split by columns: CTA r supplies columns 256 j + 128 r + (0..127),
// the slab pair m = 2 j + r (two 64-column slabs, 16 KiB).  A CTA keeps the
// pairs of its own page that it supplies (m mod 2 = r).  Into the double
// slot of each other pair m it fetches, once the scores have read it, the
// other page's pair m ^ 1 (an L2 hit: the other CTA has just loaded that
// page).  Either way the double slot of pair m feeds the P V steps of page
// m mod 2.  The rows of D that a pair MMA leaves in one CTA's TMEM sit in
// 128 lanes x N/2 columns: lane l holds head 64 r + (l mod 64), lanes 0..63
// the first half of the N columns and lanes 64..127 the second.
//
// Barriers are per tile (a ring of 4): the value-slab loads of a tile (both
// CTAs) complete two (pairs 0-1 and 2-3), its score MMAs commit one per pair
// (so each pair's reload starts as soon as the scores have read it), its
// value reloads complete one and its P V commits one; the issuing threads
// otherwise issue MMAs back to back.
//
// Pipeline: the score MMAs of tile i + 1 are issued as soon as the softmax
// of tile i has copied the scores to registers (freeing them), and P V of
// tile i as soon as its P is written, by a second issuing warp: the tensor
// pipe interleaves the two.  Before the softmax of tile i writes P or
// rescales O it waits for P V of tile i - 1.
//
// Warp roles (384 threads per CTA, each role on whole warps with one lane
// issuing): warp 0 issues the score-side TMA loads and warp 10 the
// value-side ones (both CTAs, counted on the leader's barriers); in the
// leader, warp 1 issues the pair's score MMAs and warp 11 its P V MMAs;
// warps 2..9 run the online softmax, one TMEM lane (a head and one page of
// the tile) and 32 score columns per thread, and write the segment's
// partial output.
//
// TMEM (512 columns): [0,64) the score tile, [64,320) the latent output
// (two 128-column blocks), [320,512) the query's latent columns 0..383 (A of
// the first 24 score K steps).
//
// Shared memory: the query's last 3 K slabs (64 heads x 64 values, 128-byte
// swizzle, K-major), P (2 pages x 64 heads x 64 tokens), a ring of 16 KiB
// double slots for the value slab pairs and a short ring of 8 KiB slots for
// the rotary slab (and, in split-query mode, the low query slabs).
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
constexpr int kPairs = kDc / 128;  // 4 value slab pairs per page; the ninth slab is the rotary key
constexpr int kSlab = 64 * 128;    // 64 rows x 64 bf16, 128-byte swizzle
// Double slots for value slab pairs (build-time tunable; the defaults fill
// the shared memory beside the query, P and the short ring).
#ifndef MLA_PAIR_VSLOTS
#define MLA_PAIR_VSLOTS 10
#endif
#ifndef MLA_PAIR_VSLOTS_SPLIT
#define MLA_PAIR_VSLOTS_SPLIT 9
#endif
constexpr int kTmemS = 0, kTmemO = 64, kTmemQ = 320, kTmemCols = 512;
constexpr int kSoftmaxWarps = 8;  // two per TMEM lane quarter, each on 32 of the tile's 64 columns
constexpr int kSoftmaxWarp0 = 2;  // warps 2..9
constexpr int kVcWarp = kSoftmaxWarp0 + kSoftmaxWarps;
constexpr int kPvWarp = kVcWarp + 1;
constexpr int kThreads = 32 * (kPvWarp + 1);
constexpr float kRescaleLog2 = 8.f;
constexpr uint16_t kBoth = 3;  // multicast mask: both CTAs of the pair

// Ring geometry.  Value pair m of tile ti is item g = 4 ti + m of the double
// slot ring; the short ring carries per tile the rotary slab, and in
// split-query mode the 9 low query slabs in K order (item k = e for the low
// slab e < 8, 8 for the rotary slab, 9 for the low slab 8).  Per-tile
// barriers form a ring of kT.
constexpr int kT = 4;
__device__ __forceinline__ int tslot(int ti) { return ti % kT; }
__device__ __forceinline__ uint32_t tpar(int ti) { return (uint32_t)(ti / kT) & 1u; }

template <bool kSplit>
struct Ring {
  static constexpr int kV = kSplit ? MLA_PAIR_VSLOTS_SPLIT : MLA_PAIR_VSLOTS;
  static constexpr int kS = kSplit ? 3 : 2;
  static constexpr int kPerTile = kSplit ? kSlabs + 1 : 1;
  static constexpr int kRope = kSplit ? 8 : 0;
  __device__ static int vslot(int ti, int m) { return (ti * kPairs + m) % kV; }
  __device__ static uint32_t vuse(int ti, int m) { return (uint32_t)((ti * kPairs + m) / kV); }
  __device__ static int lo_item(int e) { return e < 2 * kPairs ? e : 9; }
  __device__ static int sslot(int ti, int k) { return (ti * kPerTile + k) % kS; }
  __device__ static uint32_t suse(int ti, int k) { return (uint32_t)((ti * kPerTile + k) / kS); }
};

// A tile's value pairs may reuse only double slots whose P V was issued before
// the tile's scores (P V runs one tile behind): at least two tiles of slots.
static_assert(Ring<false>::kV >= 2 * kPairs && Ring<true>::kV >= 2 * kPairs, "too few double slots");

template <bool kSplit>
struct Smem {
  using R = Ring<kSplit>;
  uint8_t q[kSmemQSlabs][kSlab];  // query K slabs 6..8; first member: 1024-byte aligned
  uint8_t p[2][kSlab];            // P of the tile: [page of the tile] 64 heads x 64 tokens
  uint8_t v[R::kV][2][kSlab];     // value slab pairs (score-side B, then P V B)
  uint8_t r[R::kS][kSlab];        // rotary slabs (and low query slabs)
  uint64_t kfull[kT][2];  // per tile and half (pairs 0-1, 2-3): value-slab loads of both CTAs
  uint64_t qkd[kT][kPairs];  // per tile and pair: the score MMAs have read the pair
  uint64_t vfull[kT], vempty[kT];  // per tile: value reloads landed, P V over
  uint64_t rfull[R::kS], rempty[R::kS];                 // short ring
  uint64_t q_full, q_empty, qt_full;
  uint64_t s_full, s_free, p_full, pv_done;
  uint64_t o_free, fin, xbar[2], lbar;  // xbar, lbar: the softmax warps' exchanges
  float xm[2][2][128];  // [tile parity][column half] partial tile max of each TMEM lane
  float xl[2][128];     // [column half] partial row sums at the end of a segment
  uint32_t tmem_base;
  int abort_flag;
};

template <bool kSplit>
constexpr size_t smem_bytes() {
  return sizeof(Smem<kSplit>) + 1024;
}
static_assert(smem_bytes<false>() <= 232448, "shared memory over the 227 KiB per-block limit");
static_assert(smem_bytes<true>() <= 232448, "shared memory over the 227 KiB per-block limit");

struct Params {
  const bf16* q;  // packed query rows [rows][H][576] (the TMEM part is read from here)
  const int32_t* block_table;
  const int32_t* seq_lens;
  int max_blocks, num_blocks, n_q;
  float scale_log2;
  unsigned long long wait_ns;
  void* ws;
  DecodeLayout L;
};

template <bool kSplit>
__device__ __forceinline__ void set_abort(Smem<kSplit>& sm) {
  *(volatile int*)&sm.abort_flag = 1;
}
template <bool kSplit>
__device__ __forceinline__ bool aborted(Smem<kSplit>& sm) {
  return *(volatile int*)&sm.abort_flag != 0;
}

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

// ---------------------------------------------------------------- warp-uniform roles
// Every role runs on whole warps; one lane issues the TMA, MMA, commit and
// expect-tx instructions.  Values that all lanes hold alike are broadcast
// from lane 0 (uni), so that they and the descriptors and coordinates built
// from them stay in the warp-uniform datapath those instructions read from
// (a value the compiler must treat as per-lane costs a slow move into it at
// every instruction whose operands changed).
__device__ __forceinline__ int uni(int x) { return __shfl_sync(0xffffffffu, x, 0); }

#ifndef MLA_SOFTMAX_SLEEP_NS
#define MLA_SOFTMAX_SLEEP_NS 0
#endif
// A warp waits with lane 0 polling while the others sit at the warp barrier
// (waiting warps do not flood the SM's shared-memory pipe); the outcome is
// the warp's.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int where, uint64_t wns, int lane,
                                          uint32_t sleep_ns = 0) {
  int ok = 1;
  if (lane == 0) ok = mbar_wait(bar, parity, where, wns, sleep_ns) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// ---------------------------------------------------------------- tiles
// Walks the worker's tiles in order: segment, first page of the tile (whole
// warps only: the segment is read once and broadcast).
struct Tiles {
  const int4* segs;
  const int32_t* seq_lens;
  int n_q;
  int si, seg_end, pg, nseg;  // nseg: segments started so far (this one included)
  int v, pg0, pg1, len;       // the segment: query row, first page, end page, visible rows
  __device__ Tiles(const int4* s, const int32_t* sl, int nq, int b, int e)
      : segs(s), seq_lens(sl), n_q(nq), si(b), seg_end(e), pg(0), nseg(1), v(0), pg0(0), pg1(0), len(0) {
    load();
    pg = pg0;
  }
  __device__ void load() {
    if (si < seg_end) {
      const int4 g = segs[si];
      v = uni(g.x);
      pg0 = uni(g.y);
      pg1 = uni(g.z);
      // query row v sees its sequence's rows up to and including its own
      len = uni(seq_lens[v / n_q] - n_q + v % n_q + 1);
    }
  }
  __device__ bool valid() const { return si < seg_end; }
  __device__ int row() const { return v; }
  __device__ int visible() const { return len; }
  __device__ bool first() const { return pg == pg0; }
  __device__ bool last() const { return pg + 2 >= pg1; }
  __device__ bool has_b() const { return pg + 1 < pg1; }
  __device__ void next() {
    pg += 2;
    if (pg >= pg1 && ++si < seg_end) {
      load();
      pg = pg0;
      ++nseg;
    }
  }
};


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

// ---------------------------------------------------------------- TMA producers
// Score-side loads (warp 0): the segment's query slabs held in shared
// memory, then per tile the 8 value slabs of this CTA's page into their
// pairs' double slots (counted on the tile's barrier), then the short-ring
// items: the rotary slab and, in split-query mode, the low query slabs (one
// barrier each).
template <bool kSplit>
__device__ void producer_k(Smem<kSplit>& sm, const CUtensorMap* pool, const CUtensorMap* qmap,
                           const CUtensorMap* qlomap, const Params& p, int seg_begin, int seg_end, uint32_t rank,
                           int lane) {
  using R = Ring<kSplit>;
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const bool lead = rank == 0, issue = lane == 0;
  const uint64_t wns = p.wait_ns;
  int nq = 0;  // query loads issued
  int ti = 0;
  for (Tiles t(segs, p.seq_lens, p.n_q, seg_begin, seg_end); t.valid() && !uni(aborted(sm) ? 1 : 0); t.next(), ++ti) {
    const int v = t.row();
    if (t.first()) {
      if (nq >= 1 && !warp_wait(&sm.q_empty, (nq - 1) & 1, 70, wns, lane)) goto fail;
      if (issue) {
        if (lead) mbar_arrive_expect_tx(&sm.q_full, 2 * kSmemQSlabs * kSlab);
        for (int e = kTmemQSlabs; e < kSlabs; ++e)
          tma_load_2d_pair(sm.q[e - kTmemQSlabs], qmap, 64 * e, v * kH + kHalfH * (int)rank, leader(&sm.q_full));
      }
      ++nq;
    }
    const bool has = rank == 0 || t.has_b();
    const int blk = t.pg + (int)rank;
    const int phys = has ? uni(phys_block(p, v, blk, true)) : 0;
    const int y = has ? page_valid(t.visible(), blk) - kBS : 0;
    const uint32_t page_bytes = (t.has_b() ? 2 : 1) * kSlab;
    // without split-query low slabs the short ring holds only rotary slabs: load it first
    if (!kSplit) {
      const int sl = R::sslot(ti, R::kRope);
      const uint32_t use = R::suse(ti, R::kRope);
      if (use >= 1 && !warp_wait(&sm.rempty[sl], (use - 1) & 1, 72, wns, lane)) goto fail;
      if (issue && lead) mbar_arrive_expect_tx(&sm.rfull[sl], page_bytes);
      if (issue && has) tma_load_3d_pair(sm.r[sl], pool, 64 * (kSlabs - 1), y, phys, leader(&sm.rfull[sl]));
    }
    // the tile barriers' previous phase (tile ti - kT) is over once that tile's scores were done
    if (ti >= kT && !warp_wait(&sm.qkd[tslot(ti)][kPairs - 1], tpar(ti - kT), 69, wns, lane)) goto fail;
    for (int e = 0; e < 2 * kPairs; ++e) {  // the 8 value slabs, on the tile's half barriers
      const int g = ti * kPairs + (e >> 1), h = e >> 2;
      if ((e & 1) == 0 && g >= R::kV) {  // the double slot's previous tile is past its P V
        const int tp = (g - R::kV) / kPairs;
        if (!warp_wait(&sm.vempty[tslot(tp)], tpar(tp), 71, wns, lane)) goto fail;
      }
      if (issue && lead && (e & 3) == 0) mbar_arrive_expect_tx(&sm.kfull[tslot(ti)][h], 4 * page_bytes);
      if (issue && has)
        tma_load_3d_pair(sm.v[g % R::kV][e & 1], pool, 64 * e, y, phys, leader(&sm.kfull[tslot(ti)][h]));
    }
    // then (split-query mode) the short-ring items in their order (the score MMAs free them one by one)
    for (int k = 0; kSplit && k < R::kPerTile; ++k) {
      const int sl = R::sslot(ti, k);
      const uint32_t use = R::suse(ti, k);
      if (use >= 1 && !warp_wait(&sm.rempty[sl], (use - 1) & 1, 72, wns, lane)) goto fail;
      if (!issue) continue;
      if (k == R::kRope) {
        if (lead) mbar_arrive_expect_tx(&sm.rfull[sl], page_bytes);
        if (has) tma_load_3d_pair(sm.r[sl], pool, 64 * (kSlabs - 1), y, phys, leader(&sm.rfull[sl]));
      } else {  // the low part of the query for K slab e
        const int e = k < 2 * kPairs ? k : kSlabs - 1;
        if (lead) mbar_arrive_expect_tx(&sm.rfull[sl], 2 * kSlab);
        tma_load_2d_pair(sm.r[sl], qlomap, 64 * e, v * kH + kHalfH * (int)rank, leader(&sm.rfull[sl]));
      }
    }
  }
  return;
fail:
  set_abort(sm);
}

// Value-side loads (warp 6): once the scores of a tile have been computed,
// for every pair m the CTA that does not supply pair m's columns fetches the
// other page's pair m ^ 1 into that double slot; the leader counts the
// tile's bytes on one barrier.
template <bool kSplit>
__device__ void producer_v(Smem<kSplit>& sm, const CUtensorMap* pool, const Params& p, int seg_begin, int seg_end,
                           uint32_t rank, int lane) {
  using R = Ring<kSplit>;
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const bool lead = rank == 0, issue = lane == 0;
  int ti = 0;
  for (Tiles t(segs, p.seq_lens, p.n_q, seg_begin, seg_end); t.valid() && !uni(aborted(sm) ? 1 : 0); t.next(), ++ti) {
    const int v = t.row(), len_v = t.visible();
    // pairs 0 and 2 read page 0, pairs 1 and 3 page 1 (absent in a one-page tile)
    if (issue && lead) mbar_arrive_expect_tx(&sm.vfull[tslot(ti)], (t.has_b() ? 4 : 2) * 2 * kSlab);
    // this CTA reloads the pairs m with m mod 2 != rank, all from page 1 - rank,
    // each once the scores have read it
    const int pgi = 1 - (int)rank;
    const bool exists = pgi == 0 || t.has_b();
    const int blk = t.pg + pgi;
    const int y = exists ? page_valid(len_v, blk) - kBS : 0, phys = exists ? uni(phys_block(p, v, blk, false)) : 0;
    for (int m = pgi; m < kPairs; m += 2) {
      if (!warp_wait(&sm.qkd[tslot(ti)][m], tpar(ti), 73, p.wait_ns, lane)) goto fail;
      const int ds = R::vslot(ti, m), x = 128 * (m ^ 1);
      if (issue && exists) {
        tma_load_3d_pair(sm.v[ds][0], pool, x, y, phys, leader(&sm.vfull[tslot(ti)]));
        tma_load_3d_pair(sm.v[ds][1], pool, x + 64, y, phys, leader(&sm.vfull[tslot(ti)]));
      }
    }
  }
  return;
fail:
  set_abort(sm);
}

// ---------------------------------------------------------------- MMA issuer (leader CTA)
// The score MMAs of tile ti over the 9 K slabs.
template <bool kSplit>
__device__ bool issue_scores(Smem<kSplit>& sm, uint32_t tmem, const Tiles& t, int ti, uint64_t wns, int lane) {
  using R = Ring<kSplit>;
  constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
  const bool issue = lane == 0;
  const uint32_t d = tmem + kTmemS;
  const int rope_sl = R::sslot(ti, R::kRope);
  // every descriptor of the tile before the waits: the MMA queue is short,
  // so arithmetic between two MMAs would leave the tensor pipe idle
  uint64_t bdesc[kSlabs];
#pragma unroll
  for (int m = 0; m < kPairs; ++m) {
    const uint64_t b0 = kmajor_desc(sm.v[R::vslot(ti, m)][0], 0);
    bdesc[2 * m] = b0;
    bdesc[2 * m + 1] = desc_add(b0, kSlab);
  }
  bdesc[kSlabs - 1] = kmajor_desc(sm.r[rope_sl], 0);
  const uint64_t qdesc = kmajor_desc(sm.q[0], 0);
  if (t.first() && (!warp_wait(&sm.q_full, (t.nseg - 1) & 1, 80, wns, lane) ||
                    !warp_wait(&sm.qt_full, (t.nseg - 1) & 1, 79, wns, lane)))
    return false;
  if (ti >= 1 && !warp_wait(&sm.s_free, (ti - 1) & 1, 81, wns, lane)) return false;
#pragma unroll
  for (int e = 0; e < kSlabs; ++e) {
    if (e == 0 || e == 4) {
      if (!warp_wait(&sm.kfull[tslot(ti)][e >> 2], tpar(ti), 82, wns, lane)) return false;
      tc_fence_after();
    }
    if (e == kSlabs - 1) {
      if (!warp_wait(&sm.rfull[rope_sl], R::suse(ti, R::kRope) & 1, 78, wns, lane)) return false;
      tc_fence_after();
    }
    const uint64_t bd = bdesc[e];
    if (e < kTmemQSlabs) {  // A (query) from TMEM: 8 columns of bf16 pairs per 16-value K step
      if (issue) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_ts_pair(d, tmem + kTmemQ + 32 * e + 8 * j, desc_add(bd, 32 * j), idesc_s, (e | j) ? 1u : 0u);
      }
    } else {
      const uint64_t ad = desc_add(qdesc, (e - kTmemQSlabs) * kSlab);
      if (issue) {
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_ss_pair(d, desc_add(ad, 32 * j), desc_add(bd, 32 * j), idesc_s, 1u);
      }
    }
    if (kSplit) {
      const int k = R::lo_item(e), lo_sl = R::sslot(ti, k);
      if (!warp_wait(&sm.rfull[lo_sl], R::suse(ti, k) & 1, 83, wns, lane)) return false;
      tc_fence_after();
      const uint64_t ad = kmajor_desc(sm.r[lo_sl], 0);
      if (issue) {
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_ss_pair(d, desc_add(ad, 32 * j), desc_add(bd, 32 * j), idesc_s, 1u);
        mma_commit_pair(&sm.rempty[lo_sl], kBoth);
      }
    }
    if (issue && (e & 1) && e < 2 * kPairs) mma_commit_pair(&sm.qkd[tslot(ti)][e >> 1], kBoth);
  }
  if (issue) {
    mma_commit_pair(&sm.rempty[rope_sl], kBoth);
    mma_commit_pair(&sm.s_full, kBoth);
    if (t.last()) mma_commit_pair(&sm.q_empty, kBoth);
  }
  __syncwarp();
  return true;
}

// P V of tile ti: latent block j, page q from the double slot of pair 2 j + q.
template <bool kSplit>
__device__ bool issue_pv(Smem<kSplit>& sm, uint32_t tmem, const Tiles& t, int ti, uint64_t wns, int lane) {
  using R = Ring<kSplit>;
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, 256, 0, 1);
  const bool issue = lane == 0;
  const bool two = t.has_b(), first = t.first();
  // the slab pairs as MN-major B operands: two 64-column groups one slab
  // apart (LBO), 8-token groups 1 KiB apart (SBO), 16 tokens per K step
  uint64_t vdesc[kPairs];
#pragma unroll
  for (int m = 0; m < kPairs; ++m) vdesc[m] = smem_desc(smem_u32(sm.v[R::vslot(ti, m)][0]), kSlab, 1024, kSwizzle128B);
  const uint64_t pdesc = kmajor_desc(sm.p[0], 0);
  if (first && t.nseg >= 2 && !warp_wait(&sm.o_free, (t.nseg - 2) & 1, 84, wns, lane)) return false;
  if (!warp_wait(&sm.p_full, ti & 1, 85, wns, lane)) return false;
  if (!warp_wait(&sm.vfull[tslot(ti)], tpar(ti), 86, wns, lane)) return false;
  tc_fence_after();
#pragma unroll
  for (int j = 0; j < 2; ++j) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      if (issue && (q == 0 || two)) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss_pair(tmem + kTmemO + 128 * j, desc_add(pdesc, q * kSlab + 32 * kk), desc_add(vdesc[2 * j + q], 2048 * kk),
                      idesc_o, (first && q == 0 && kk == 0) ? 0u : 1u);
      }
    }
  }
  if (issue) {
    mma_commit_pair(&sm.vempty[tslot(ti)], kBoth);
    mma_commit_pair(&sm.pv_done, kBoth);
  }
  __syncwarp();
  return true;
}

// The two MMA issuers of the pair (leader CTA): warp 1 issues the scores of
// every tile, warp 7 the P V of every tile as soon as its P is written, so
// that the tensor pipe interleaves the two streams (P V of tile i runs among
// the scores of tile i + 1) and neither stream's waits stall the other.  A
// commit tracks the MMAs of the thread that issues it, so each stream's
// barriers see only its own MMAs.  Both end on `fin` (count 2).
template <bool kSplit>
__device__ void score_issuer(Smem<kSplit>& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end, int lane) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const uint64_t wns = p.wait_ns;
  int ti = 0;
  bool ok = true;
  for (Tiles t(segs, p.seq_lens, p.n_q, seg_begin, seg_end); t.valid() && ok; t.next(), ++ti) ok = issue_scores(sm, tmem, t, ti, wns, lane);
  if (!ok) set_abort(sm);
  if (lane == 0) mma_commit_pair(&sm.fin, 1);
  warp_wait(&sm.fin, 0, 87, wns, lane);
}

template <bool kSplit>
__device__ void pv_issuer(Smem<kSplit>& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end, int lane) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const uint64_t wns = p.wait_ns;
  int ti = 0;
  bool ok = true;
  for (Tiles t(segs, p.seq_lens, p.n_q, seg_begin, seg_end); t.valid() && ok; t.next(), ++ti) ok = issue_pv(sm, tmem, t, ti, wns, lane);
  if (!ok) set_abort(sm);
  if (lane == 0) mma_commit_pair(&sm.fin, 1);
  warp_wait(&sm.fin, 0, 88, wns, lane);
}

// ---------------------------------------------------------------- softmax

// The query's latent columns 0..383 of this lane's head into TMEM (the A
// operand of the first 24 score K steps); the two warps of a lane quarter
// take 192 columns each.  A pair MMA with A in TMEM reads each CTA's 64 rows
// from lanes 0..63 and again from lanes 64..127, so lanes l and l ^ 64 both
// hold head 64 r + (l mod 64).  Then the leader is told.
template <bool kSplit>
__device__ __forceinline__ void load_query_tmem(Smem<kSplit>& sm, const Params& p, int v, int head, uint32_t tl,
                                                int ch, int lane) {
  constexpr int kCols = kTmemQSlabs * 32 / 2;  // TMEM columns per warp (bf16 pairs): 96
  static_assert(kCols % 32 == 0, "query columns per warp in rounds of 32");
  const uint4* src = reinterpret_cast<const uint4*>(p.q + ((long long)v * kH + head) * kRow) + ch * (kCols / 4);
#pragma unroll 1
  for (int b = 0; b < kCols / 32; ++b) {  // 8 loads in flight per round, 32 columns each
    uint4 w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = __ldg(src + b * 8 + i);
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const uint32_t x[16] = {w[4 * c].x,     w[4 * c].y,     w[4 * c].z,     w[4 * c].w,
                              w[4 * c + 1].x, w[4 * c + 1].y, w[4 * c + 1].z, w[4 * c + 1].w,
                              w[4 * c + 2].x, w[4 * c + 2].y, w[4 * c + 2].z, w[4 * c + 2].w,
                              w[4 * c + 3].x, w[4 * c + 3].y, w[4 * c + 3].z, w[4 * c + 3].w};
      tmem_st16(tl + kTmemQ + ch * kCols + b * 32 + c * 16, x);
    }
  }
  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive_remote(leader(&sm.qt_full));
}

// Online softmax, one TMEM lane (a head and a page of the tile) and 32 of
// its 64 score columns per thread: warp w handles lane quarter w mod 4 and
// column half ch.  The row max and (at the end of a segment) the row sum of
// a head combine the four threads of its two lanes and two halves through
// shared memory and an mbarrier of the softmax warps (a bounded wait).

template <bool kSplit>
__device__ void softmax_role(Smem<kSplit>& sm, uint32_t tmem, const Params& p, int seg_begin, int seg_end,
                             uint32_t rank, int warp, int lane) {
  const int4* segs = ws_at<int4>(p.ws, p.L.off_seg);
  const int qw = warp & 3;                                 // TMEM lane quarter
  const int ch = (warp - kSoftmaxWarp0) >> 2;              // column half of the tile / of O
  const int l = qw * 32 + lane;                            // TMEM lane
  const int half = l >> 6;                                 // page of the tile / column half of each O block
  const int hl = l & 63, head = kHalfH * (int)rank + hl;   // head of this lane
  const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);  // this warp's lane quarter
  const uint64_t wns = p.wait_ns;
  bf16* part_o = ws_at<bf16>(p.ws, p.L.off_o);
  float* part_lse = ws_at<float>(p.ws, p.L.off_lse);

  float m_used = -INFINITY, lsum = 0.f;
  int nseg_done = 0;
  Tiles t(segs, p.seq_lens, p.n_q, seg_begin, seg_end);
  if (t.valid()) load_query_tmem(sm, p, t.row(), head, tl, ch, lane);
  for (int i = 0; t.valid(); ++i, t.next()) {
    const bool first = t.first(), last = t.last();
    if (first) {
      m_used = -INFINITY;
      lsum = 0.f;
    }
    // this lane's page: rows past the visible length sit at the top of the tile
    const int shift = kBS - ((half == 0 || t.has_b()) ? page_valid(t.visible(), t.pg + half) : 0) - 32 * ch;
    if (!warp_wait(&sm.s_full, i & 1, 90, wns, lane, MLA_SOFTMAX_SLEEP_NS)) goto fail;
    tc_fence_after();
    float s[32];
    {
      uint32_t a[32];
      tmem_ld32(tl + kTmemS + 32 * ch, a);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(a[c]);
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_remote(leader(&sm.s_free));

    float m8[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) m8[c] = -INFINITY;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      s[c] = c >= shift ? s[c] * p.scale_log2 : -INFINITY;
      m8[c & 7] = fmaxf(m8[c & 7], s[c]);
    }
    const float m_loc =
        fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
    sm.xm[i & 1][ch][l] = m_loc;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.xbar[i & 1]);
    if (!warp_wait(&sm.xbar[i & 1], (i >> 1) & 1, 91, wns, lane)) goto fail;
    const float m_tile = fmaxf(fmaxf(sm.xm[i & 1][0][l], sm.xm[i & 1][1][l]),
                               fmaxf(sm.xm[i & 1][0][l ^ 64], sm.xm[i & 1][1][l ^ 64]));

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
    uint32_t pk[16];
    float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const float p0 = fast_exp2(s[2 * c] - mbase), p1 = fast_exp2(s[2 * c + 1] - mbase);
      ps[c & 3] += p0 + p1;
      pk[c] = pack_bf16x2(p0, p1);
    }
    lsum = lsum * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));

    // P V of the previous tile reads P and accumulates into O: both must be
    // over before this tile rescales O or overwrites P.
    if (i >= 1 && !warp_wait(&sm.pv_done, (i - 1) & 1, 92, wns, lane)) goto fail;
    tc_fence_after();
    // tcgen05.ld / st are warp-collective: the warp rescales (its 4 of the
    // lane's 8 O chunks) when any lane needs it.
    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
      for (int c = 4 * ch; c < 4 * ch + 4; ++c) {
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
      // row hl of this page's P slab, K-major with the 128-byte swizzle:
      // 16-byte chunks 4 ch .. 4 ch + 3
      uint8_t* row = sm.p[half] + hl * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(row + (((4 * ch + c) ^ (hl & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_remote(leader(&sm.p_full));

    // The scores of this segment are all done (s_full of its last tile): the
    // next segment's query can replace this one in TMEM before the epilogue.
    if (last && t.si + 1 < seg_end) load_query_tmem(sm, p, segs[t.si + 1].x, head, tl, ch, lane);

    if (last) {
      // epilogue of the segment: O / l and the log2-sum-exp
      sm.xl[ch][l] = lsum;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.lbar);
      if (!warp_wait(&sm.lbar, nseg_done & 1, 94, wns, lane)) goto fail;
      const float ltot = (sm.xl[0][l] + sm.xl[1][l]) + (sm.xl[0][l ^ 64] + sm.xl[1][l ^ 64]);
      if (!warp_wait(&sm.pv_done, i & 1, 95, wns, lane)) goto fail;
      tc_fence_after();
      const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
      const int si = t.si;
      // partial output [segment][head][d] in bf16: O block j holds latent
      // columns 256 j + 128 half + (0..127) in this lane; this warp writes
      // block ch
#pragma unroll 1
      for (int c = 4 * ch; c < 4 * ch + 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tl + kTmemO + c * 32, o);
        tmem_wait_ld();
        const int d0 = 256 * (c >> 2) + 128 * half + 32 * (c & 3);
        uint4* out = reinterpret_cast<uint4*>(part_o + ((long long)si * kH + head) * kDc + d0);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float* f = reinterpret_cast<const float*>(o) + 8 * k;
          out[k] = make_uint4(pack_bf16x2(f[0] * inv, f[1] * inv), pack_bf16x2(f[2] * inv, f[3] * inv),
                              pack_bf16x2(f[4] * inv, f[5] * inv), pack_bf16x2(f[6] * inv, f[7] * inv));
        }
      }
      if (half == 0 && ch == 0) part_lse[(long long)si * kH + head] = ltot > 0.f ? m_used + log2f(ltot) : -INFINITY;
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
template <bool kSplit>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_pair_kernel(const __grid_constant__ CUtensorMap pool, const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap qlomap, const Params p) {
  using R = Ring<kSplit>;
  extern __shared__ uint8_t smem_raw[];
  Smem<kSplit>& sm =
      *reinterpret_cast<Smem<kSplit>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int worker = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kT; ++s) {
      for (int h = 0; h < 2; ++h) mbar_init(&sm.kfull[s][h], 1);
      for (int m = 0; m < kPairs; ++m) mbar_init(&sm.qkd[s][m], 1);
      mbar_init(&sm.vfull[s], 1);
      mbar_init(&sm.vempty[s], 1);
    }
    for (int s = 0; s < R::kS; ++s) {
      mbar_init(&sm.rfull[s], 1);
      mbar_init(&sm.rempty[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, 2 * kSoftmaxWarps);
    mbar_init(&sm.p_full, 2 * kSoftmaxWarps);
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    mbar_init(&sm.qt_full, 2 * kSoftmaxWarps);
    mbar_init(&sm.o_free, 2 * kSoftmaxWarps);
    for (int b = 0; b < 2; ++b) mbar_init(&sm.xbar[b], kSoftmaxWarps);
    mbar_init(&sm.lbar, kSoftmaxWarps);
    mbar_init(&sm.fin, 2);
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
    if (kSplit) prefetch_tensormap(&qlomap);
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
    seg_begin = uni(wfirst[worker]);
    seg_end = uni(wfirst[worker + 1]);
  }

  if (warp == 0) {
    producer_k(sm, &pool, &qmap, &qlomap, p, seg_begin, seg_end, rank, lane);
  } else if (warp == 1) {
    if (rank == 0) score_issuer(sm, tmem, p, seg_begin, seg_end, lane);
  } else if (warp == kPvWarp) {
    if (rank == 0) pv_issuer(sm, tmem, p, seg_begin, seg_end, lane);
  } else if (warp == kVcWarp) {
    producer_v(sm, &pool, p, seg_begin, seg_end, rank, lane);
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
  return c->dtype == MLA_BF16 && !(c->flags & MLA_FLAG_FP8_CACHE) && c->n_heads == kH && c->d_c == kDc &&
         c->d_r == kDr && c->block_size == kBS;
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
                         unsigned long long wait_ns, cudaStream_t s, bool planned = false) {
  const bool split = (c->flags & MLA_FLAG_SPLIT_QUERY) != 0;
  const long long rows = (long long)L.batch * L.n_q;
  bf16* qpack = q_packed ? const_cast<bf16*>(q_packed) : reinterpret_cast<bf16*>(static_cast<char*>(ws) + L.off_qpack);
  bf16* qlo = split ? qpack + rows * kH * kRow : nullptr;
  CUtensorMap pmap, qmap, qlomap;
  mla_status st = pool_map(k, &pmap);
  if (st == MLA_OK) st = query_map(qpack, rows, &qmap);
  if (st == MLA_OK) st = query_map(split ? qlo : qpack, rows, &qlomap);
  if (st != MLA_OK) return st;

  static std::atomic<uint64_t> plan_attr{0}, plan_only_attr{0}, dec_attr{0}, dec_split_attr{0};
  const size_t plan_smem = sizeof(int) * ((size_t)rows + 1);
  const void* dec_fn = split ? (const void*)decode_pair_kernel<true> : (const void*)decode_pair_kernel<false>;
  const size_t dec_smem = split ? smem_bytes<true>() : smem_bytes<false>();
  if (set_smem_once(dec_fn, dec_smem, split ? dec_split_attr : dec_attr) != MLA_OK) return MLA_ERR_CUDA;
  if (q_packed) {
    if (!planned) {
      if (plan_smem > 48 * 1024 &&
          set_smem_once((const void*)decode_plan_kernel, plan_smem, plan_only_attr) != MLA_OK)
        return MLA_ERR_CUDA;
      if (launch_chained(decode_plan_kernel, dim3(1), dim3(1024), plan_smem, s, seq_lens, c->block_size,
                         k->max_blocks_per_seq, ws, L) != cudaSuccess)
        return MLA_ERR_CUDA;
    }
  } else {
    if (plan_smem > 48 * 1024 && set_smem_once((const void*)pair_plan_pack_kernel, plan_smem, plan_attr) != MLA_OK)
      return MLA_ERR_CUDA;
    const long long groups = rows * kH * (kRow / 8);
    const int qblocks = (int)std::min<long long>((groups + 1023) / 1024, 4096);
    if (launch_chained(pair_plan_pack_kernel, dim3(1 + qblocks), dim3(1024), plan_smem, s, seq_lens, c->block_size,
                       k->max_blocks_per_seq, ws, L, q_lat, q_rope, rows * kH, qpack, qlo) != cudaSuccess)
      return MLA_ERR_CUDA;
  }
  const Params p{qpack,    k->block_table, seq_lens, k->max_blocks_per_seq, k->num_blocks, n_q,
                 scale * 1.4426950408889634f, wait_ns, ws, L};
  const cudaError_t e =
      split ? launch_chained(decode_pair_kernel<true>, dim3(2 * L.workers), dim3(kThreads), dec_smem, s, pmap, qmap,
                             qlomap, p)
            : launch_chained(decode_pair_kernel<false>, dim3(2 * L.workers), dim3(kThreads), dec_smem, s, pmap, qmap,
                             qlomap, p);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace pairdec
}  // namespace mla
