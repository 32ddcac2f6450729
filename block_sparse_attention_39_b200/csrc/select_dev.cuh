// Device code of a4 + a5 (local Top-K selection inside the sliding window and
// assembly of the attended-block list), shared by the per-call kernel
// (select.cu) and the fused routing kernel (route.cu).
//
// Sparse Forcing restricts attention inside the recent window to the Top-K
// blocks most relevant to each query (gist.science/es, section 2
// "Arquitectura Propuesta", item "Ventana Local") and attends the persistent
// memory densely (PBSA item "Atención Híbrida").
//
// One warp per (b, h, query block): the window's scores become 64-bit keys
// (orderable score, ~id), a warp-wide bitonic sort over the keys held in
// registers (up to 512 keys) picks the Top-K, and a second bitonic sort merges
// the selection with the memory ids into an ascending, duplicate-free list.
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

// Optional time stamps inside select_row for schedule studies (the fused
// routing kernel defines this when built with -DPBSA_ROUTE_TRACE).
#ifndef SEL_TRACE
#define SEL_TRACE(i, bh, k) do {} while (0)
#endif

namespace pbsa {
namespace dev {

constexpr int KPL = 16;                 // capacity: 512 keys per warp

// W: keys per lane of the window sort; U: keys per lane of the union sort
// (32*W >= n_win, 32*U >= n_mem + min(k, n_win)); both <= KPL.
struct SelArgs {
  const float* scores;
  const int32_t* win_ids;
  const int32_t* mem_ids;
  const int32_t* blk_len;
  const int32_t* blk_pos;
  int32_t* idx;
  int32_t* cnt;
  int* status;
  int nQB, NB, n_win, k, n_mem, mem_ld, mask, q_pos0, Tq, qc, bs, Amax, qb_offset, nQB_total;
  // Optional (NULL in the per-call kernel): lengths and positions of ids
  // 0..n_slot-1 taken from here (row bh at bh * slot_ld) instead of blk_len /
  // blk_pos -- the fused routing kernel passes the values its memory update
  // is writing, so the lists need not wait for the slot copies.
  const int32_t* slot_len;
  const int32_t* slot_pos;
  long slot_ld;
  int n_slot;
};

// Length (and position) of block id j of head bh as the selection reads them.
__device__ __forceinline__ int sel_len(const SelArgs& a, long bh, int j) {
  return (a.slot_len != nullptr && j < a.n_slot) ? a.slot_len[bh * a.slot_ld + j]
                                                 : a.blk_len[bh * a.NB + j];
}
__device__ __forceinline__ int sel_pos(const SelArgs& a, long bh, int j) {
  return (a.slot_len != nullptr && j < a.n_slot) ? a.slot_pos[bh * a.slot_ld + j]
                                                 : a.blk_pos[bh * a.NB + j];
}

// No-op hook for select_row.
struct NoWait {
  __device__ bool operator()() const { return true; }
};

// The attended list of query block i of head bh, computed by one warp.
// `before_mem()` is called by every lane after the window's Top-K is sorted
// and before any memory id's length is read; it returns false (warp-uniform)
// to abandon the row.  The fused routing kernel waits there for the memory
// update's plan, which states the slots' lengths; with slot lengths taken from
// the plan, a window id below n_slot also waits, so its length is read after
// the hook as well.
template <int W, int U, typename Hook = NoWait>
__device__ __forceinline__ void select_row(const SelArgs& a, int i, long bh,
                                           Hook before_mem = Hook()) {
  // plain pointers, no __restrict__: in the fused routing kernel the scores
  // and block lengths are written earlier in the same launch, so they must not
  // be read through the read-only data path
  const float* scores = a.scores;
  const int32_t* win_ids = a.win_ids;
  const int32_t* mem_ids = a.mem_ids;
  int32_t* idx = a.idx;
  int32_t* cnt = a.cnt;
  int* status = a.status;
  const int NB = a.NB, n_win = a.n_win, k = a.k, n_mem = a.n_mem, mem_ld = a.mem_ld;
  const int mask = a.mask, q_pos0 = a.q_pos0, Tq = a.Tq, qc = a.qc, bs = a.bs;
  const int Amax = a.Amax, qb_offset = a.qb_offset, nQB_total = a.nQB_total;
  const int lane = threadIdx.x & 31;
  const float* srow = scores + (bh * nQB_total + qb_offset + i) * static_cast<long>(NB);
  int qrow0, qlen;
  qb_rows(i, Tq, qc, bs, qrow0, qlen);
  const int last_q = q_pos0 + qrow0 + qlen - 1;

  // ---- gather: window ids and memory ids first, then their lengths/scores,
  // so each lane has all of its loads in flight at once.  Memory entry e is
  // held at union element 32*U-1-e: the top `take` selected keys occupy
  // elements [0, take) of the union and take + n_mem <= 32*U, so the two
  // never collide.
  int wid[W], mid[U];
#pragma unroll
  for (int r = 0; r < W; ++r) {
    const int e = lane + 32 * r;               // coalesced over lanes
    wid[r] = e < n_win ? win_ids[e] : -1;
  }
#pragma unroll
  for (int r = 0; r < U; ++r) {
    const int me = 32 * U - 1 - (lane * U + r);
    mid[r] = me < n_mem ? mem_ids[bh * mem_ld + me] : -1;
  }
  // ---- Top-K over the window (element order is irrelevant before the sort)
  uint64_t wkey[W];
  int n_ok = 0;
  auto window_topk = [&]() {
    int wlen[W], wpos[W];
    float wsc[W];
#pragma unroll
    for (int r = 0; r < W; ++r) {
      const int j = wid[r];
      const bool in = j >= 0 && j < NB;
      if (r * 32 + lane < n_win && !in) report_status(status, PBSA_ERR_ARG);
      wlen[r] = in ? sel_len(a, bh, j) : 0;
      wsc[r] = in ? srow[j] : 0.f;
      wpos[r] = (in && mask == PBSA_MASK_TOKEN) ? sel_pos(a, bh, j) : 0;
    }
    n_ok = 0;
#pragma unroll
    for (int r = 0; r < W; ++r) {
      bool ok = wlen[r] > 0;
      if (mask == PBSA_MASK_TOKEN) ok = ok && wpos[r] <= last_q;
      wkey[r] = ok ? score_key(wsc[r], static_cast<uint32_t>(wid[r])) : 0ull;
      n_ok += ok ? 1 : 0;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) n_ok += __shfl_xor_sync(0xffffffffu, n_ok, off);
    warp_bitonic_sort_desc<W>(wkey);
  };
  bool win_late = false;
  if (a.slot_len != nullptr) {
    bool low = false;
#pragma unroll
    for (int r = 0; r < W; ++r) low = low || (wid[r] >= 0 && wid[r] < a.n_slot);
    win_late = __any_sync(0xffffffffu, low);
  }
  SEL_TRACE(i, bh, 0);
  if (!win_late) window_topk();
  SEL_TRACE(i, bh, 1);
  if (!before_mem()) return;
  SEL_TRACE(i, bh, 2);
  if (win_late) window_topk();
  const int take = min(k, n_ok);
  int mlen[U];
#pragma unroll
  for (int r = 0; r < U; ++r) {
    const int m = mid[r];
    // -1 names no block; any other id outside the pool is an argument error
    if (m >= NB || m < -1) report_status(status, PBSA_ERR_ARG);
    mlen[r] = (m >= 0 && m < NB) ? sel_len(a, bh, m) : 0;
  }

  // ---- union with the memory ids, ascending (descending sort of ~id).
  // Sorted window element e (lane e / W, register e % W) moves to union
  // element e (lane e / U, register e % U) through one shuffle per register.
  uint64_t key[U];
#pragma unroll
  for (int r = 0; r < U; ++r) {
    const int e = lane * U + r;                      // union element held here
    const int src_lane = (e / W) & 31, src_reg = e % W;
    uint64_t got = 0;
#pragma unroll
    for (int q = 0; q < W; ++q) {
      const uint64_t v = __shfl_sync(0xffffffffu, wkey[q], src_lane);
      if (q == src_reg) got = v;
    }
    uint64_t nk = 0;
    if (e < take) {
      nk = 0xffffffffull - key_id(got);
    } else if (mid[r] >= 0 && mid[r] < NB && mlen[r] > 0) {
      nk = 0xffffffffull - static_cast<uint32_t>(mid[r]);
    }
    key[r] = nk;
  }
  SEL_TRACE(i, bh, 3);
  warp_bitonic_sort_desc<U>(key);
  SEL_TRACE(i, bh, 4);

  // ---- dedupe and write
  uint64_t prev_last = __shfl_up_sync(0xffffffffu, key[U - 1], 1);
  int keep[U];
  int mine = 0;
#pragma unroll
  for (int r = 0; r < U; ++r) {
    const uint64_t prev = (r == 0) ? ((lane == 0) ? ~0ull : prev_last) : key[r - 1];
    keep[r] = (key[r] != 0 && key[r] != prev) ? 1 : 0;
    mine += keep[r];
  }
  int incl = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  int pos = incl - mine;
  int32_t* out = idx + (bh * nQB_total + qb_offset + i) * static_cast<long>(Amax);
  if (total > Amax) {
    // the list does not fit: report it and leave an empty, defined list so
    // that a later attention call on the same stream attends nothing rather
    // than a previous call's blocks
    if (lane == 0) report_status(status, PBSA_ERR_SHAPE);
    for (int e = lane; e < Amax; e += 32) out[e] = -1;
    if (lane == 0) cnt[bh * nQB_total + qb_offset + i] = 0;
    return;
  }
#pragma unroll
  for (int r = 0; r < U; ++r) {
    if (keep[r]) out[pos++] = static_cast<int32_t>(0xffffffffu - static_cast<uint32_t>(key[r]));
  }
  for (int e = total + lane; e < Amax; e += 32) out[e] = -1;
  if (lane == 0) cnt[bh * nQB_total + qb_offset + i] = total;
  SEL_TRACE(i, bh, 5);
}

// Shared memory per warp of select_row_bitmap: 32*W window keys and a bitmap
// of kSelBmWords words (block ids below 32 * kSelBmWords).
constexpr int kSelBmWords = 1024;
template <int W>
__host__ __device__ constexpr int sel_bitmap_smem_per_warp() {
  return 32 * W * 8 + kSelBmWords * 4;
}

// The same list as select_row, computed without sorting: the window's Top-K
// by counting, for each candidate, the keys larger than its own (keys are
// unique: the id is in the low bits), and the union with the memory ids as a
// bitmap over block ids, emitted in ascending order with a popcount prefix
// scan (duplicates merge in the bitmap).  Needs NB <= 32 * kSelBmWords.
// `wsm` is this warp's shared memory (sel_bitmap_smem_per_warp<W>() bytes).
template <int W, int U, typename Hook = NoWait>
__device__ __forceinline__ void select_row_bitmap(const SelArgs& a, int i, long bh, uint8_t* wsm,
                                                  Hook before_mem = Hook()) {
  uint64_t* skeys = reinterpret_cast<uint64_t*>(wsm);                 // [32*W]
  uint32_t* bm = reinterpret_cast<uint32_t*>(wsm + 32 * W * 8);       // [kSelBmWords]
  const int NB = a.NB, n_win = a.n_win, n_mem = a.n_mem;
  const int lane = threadIdx.x & 31;
  const float* srow = a.scores + (bh * a.nQB_total + a.qb_offset + i) * static_cast<long>(NB);
  int qrow0, qlen;
  qb_rows(i, a.Tq, a.qc, a.bs, qrow0, qlen);
  const int last_q = a.q_pos0 + qrow0 + qlen - 1;
  const int nbw = (NB + 31) / 32;

  int wid[W], mid[U];
#pragma unroll
  for (int r = 0; r < W; ++r) {
    const int e = lane + 32 * r;
    wid[r] = e < n_win ? a.win_ids[e] : -1;
  }
#pragma unroll
  for (int r = 0; r < U; ++r) {
    const int me = lane + 32 * r;
    mid[r] = me < n_mem ? a.mem_ids[bh * a.mem_ld + me] : -1;
  }
  // the bitmap starts empty
  for (int w = lane; w < nbw; w += 32) bm[w] = 0u;
  uint64_t wkey[W];
  bool wsel[W];
  auto window_topk = [&]() {
    int n_ok = 0;
#pragma unroll
    for (int r = 0; r < W; ++r) {
      const int j = wid[r];
      const bool in = j >= 0 && j < NB;
      if (r * 32 + lane < n_win && !in) report_status(a.status, PBSA_ERR_ARG);
      const int len = in ? sel_len(a, bh, j) : 0;
      const float sc = in ? srow[j] : 0.f;
      const int pos = (in && a.mask == PBSA_MASK_TOKEN) ? sel_pos(a, bh, j) : 0;
      bool ok = len > 0;
      if (a.mask == PBSA_MASK_TOKEN) ok = ok && pos <= last_q;
      wkey[r] = ok ? score_key(sc, static_cast<uint32_t>(j)) : 0ull;
      skeys[lane + 32 * r] = wkey[r];
      n_ok += __popc(__ballot_sync(0xffffffffu, ok));
    }
    __syncwarp();
    const int take = min(a.k, n_ok);
    // rank = number of larger keys; two keys per 16-byte shared load
    int rank[W];
#pragma unroll
    for (int r = 0; r < W; ++r) rank[r] = 0;
    const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(skeys);
#pragma unroll 4
    for (int f = 0; f < 16 * W; ++f) {
      const ulonglong2 v = k2[f];
#pragma unroll
      for (int r = 0; r < W; ++r) rank[r] += (v.x > wkey[r] ? 1 : 0) + (v.y > wkey[r] ? 1 : 0);
    }
#pragma unroll
    for (int r = 0; r < W; ++r) wsel[r] = wkey[r] != 0ull && rank[r] < take;
  };
  bool win_late = false;
  if (a.slot_len != nullptr) {
    bool low = false;
#pragma unroll
    for (int r = 0; r < W; ++r) low = low || (wid[r] >= 0 && wid[r] < a.n_slot);
    win_late = __any_sync(0xffffffffu, low);
  }
  SEL_TRACE(i, bh, 0);
  if (!win_late) window_topk();
  SEL_TRACE(i, bh, 1);
  if (!before_mem()) return;
  SEL_TRACE(i, bh, 2);
  if (win_late) window_topk();
  __syncwarp();                               // the bitmap is zero
#pragma unroll
  for (int r = 0; r < W; ++r)
    if (wsel[r]) atomicOr(&bm[wid[r] >> 5], 1u << (wid[r] & 31));
#pragma unroll
  for (int r = 0; r < U; ++r) {
    const int m = mid[r];
    // -1 names no block; any other id outside the pool is an argument error
    if (m >= NB || m < -1) report_status(a.status, PBSA_ERR_ARG);
    if (m >= 0 && m < NB && sel_len(a, bh, m) > 0) atomicOr(&bm[m >> 5], 1u << (m & 31));
  }
  __syncwarp();
  SEL_TRACE(i, bh, 3);
  // ---- count, then write the ids in ascending order
  int total = 0;
  for (int w0 = 0; w0 < nbw; w0 += 32) {
    const uint32_t word = w0 + lane < nbw ? bm[w0 + lane] : 0u;
    int c = __popc(word);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
    total += c;
  }
  int32_t* out = a.idx + (bh * a.nQB_total + a.qb_offset + i) * static_cast<long>(a.Amax);
  int32_t* cnt = a.cnt + bh * a.nQB_total + a.qb_offset + i;
  if (total > a.Amax) {
    if (lane == 0) report_status(a.status, PBSA_ERR_SHAPE);
    for (int e = lane; e < a.Amax; e += 32) out[e] = -1;
    if (lane == 0) *cnt = 0;
    return;
  }
  int base = 0;
  for (int w0 = 0; w0 < nbw; w0 += 32) {
    uint32_t word = w0 + lane < nbw ? bm[w0 + lane] : 0u;
    const int c = __popc(word);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int pos = base + incl - c;
    while (word) {
      const int b = __ffs(word) - 1;
      out[pos++] = (w0 + lane) * 32 + b;
      word &= word - 1u;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  for (int e = total + lane; e < a.Amax; e += 32) out[e] = -1;
  if (lane == 0) *cnt = total;
  SEL_TRACE(i, bh, 4);
  SEL_TRACE(i, bh, 5);
}

// Shared memory per warp of select_row_hier: that of select_row_bitmap plus
// the window's per-entry (weighted score, length, frame) for the frame scores.
template <int W>
__host__ __device__ constexpr int sel_hier_smem_per_warp() {
  return sel_bitmap_smem_per_warp<W>() + 32 * W * 12;
}

// The two-level local selection (frame, then block) for query block i of head
// bh, computed by one warp; the list is the union with the memory ids as in
// select_row.  Light Forcing keeps, per query block, a few relevant frames by
// frame-level pooled keys and then the critical blocks inside them by
// block-level keys (gist.science/it, section 2.2 "Attenzione Sparsa
// Gerarchica (HSA)").  Here a frame is a group of window blocks (win_frame[e]
// is the frame of window entry e, 0 <= label < n_frames <= 32); its score is
// the length-weighted mean of its candidate blocks' scores (its pooled key is
// the mean of its blocks' tokens and scores are linear in the key), summed in
// window order; the F frames of highest score are kept (ties: lower label) and
// the Top-K blocks of the kept frames are taken as in select_row_bitmap.
template <int W, int U>
__device__ __forceinline__ void select_row_hier(const SelArgs& a, const int32_t* win_frame,
                                                int n_frames, int F, int i, long bh,
                                                uint8_t* wsm) {
  uint64_t* skeys = reinterpret_cast<uint64_t*>(wsm);                 // [32*W]
  uint32_t* bm = reinterpret_cast<uint32_t*>(wsm + 32 * W * 8);       // [kSelBmWords]
  float* f_num = reinterpret_cast<float*>(wsm + sel_bitmap_smem_per_warp<W>());  // [32*W]
  float* f_den = f_num + 32 * W;                                      // [32*W]
  int* f_lab = reinterpret_cast<int*>(f_den + 32 * W);                // [32*W]
  const int NB = a.NB, n_win = a.n_win, n_mem = a.n_mem;
  const int lane = threadIdx.x & 31;
  const float* srow = a.scores + (bh * a.nQB_total + a.qb_offset + i) * static_cast<long>(NB);
  int qrow0, qlen;
  qb_rows(i, a.Tq, a.qc, a.bs, qrow0, qlen);
  const int last_q = a.q_pos0 + qrow0 + qlen - 1;
  const int nbw = (NB + 31) / 32;

  int wid[W], wfr[W], mid[U];
#pragma unroll
  for (int r = 0; r < W; ++r) {
    const int e = lane + 32 * r;
    wid[r] = e < n_win ? a.win_ids[e] : -1;
    wfr[r] = e < n_win ? win_frame[e] : -1;
  }
#pragma unroll
  for (int r = 0; r < U; ++r) {
    const int me = lane + 32 * r;
    mid[r] = me < n_mem ? a.mem_ids[bh * a.mem_ld + me] : -1;
  }
  for (int w = lane; w < nbw; w += 32) bm[w] = 0u;
  // ---- candidates of the window, and their frames' weighted scores
  uint64_t wkey[W];
#pragma unroll
  for (int r = 0; r < W; ++r) {
    const int j = wid[r];
    const int e = lane + 32 * r;
    const bool in = j >= 0 && j < NB;
    if (e < n_win && !in) report_status(a.status, PBSA_ERR_ARG);
    const bool lab_ok = wfr[r] >= 0 && wfr[r] < n_frames;
    if (e < n_win && !lab_ok) report_status(a.status, PBSA_ERR_ARG);
    const int len = in ? sel_len(a, bh, j) : 0;
    const float sc = in ? srow[j] : 0.f;
    const int pos = (in && a.mask == PBSA_MASK_TOKEN) ? sel_pos(a, bh, j) : 0;
    bool ok = len > 0 && lab_ok;
    if (a.mask == PBSA_MASK_TOKEN) ok = ok && pos <= last_q;
    wkey[r] = ok ? score_key(sc, static_cast<uint32_t>(j)) : 0ull;
    f_num[e] = ok ? static_cast<float>(len) * sc : 0.f;
    f_den[e] = ok ? static_cast<float>(len) : 0.f;
    f_lab[e] = ok ? wfr[r] : -1;
  }
  __syncwarp();
  // lane g sums frame g over the window in order
  float num = 0.f, den = 0.f;
  if (lane < n_frames) {
    for (int e = 0; e < n_win; ++e) {
      if (f_lab[e] == lane) {
        num += f_num[e];
        den += f_den[e];
      }
    }
  }
  const bool has = den > 0.f;
  const float fs = has ? num / den : -INFINITY;
  int frank = 0;
#pragma unroll 4
  for (int m = 0; m < 32; ++m) {
    const float o = __shfl_sync(0xffffffffu, fs, m);
    const bool oh = __shfl_sync(0xffffffffu, has, m);
    frank += (oh && (o > fs || (o == fs && m < lane))) ? 1 : 0;
  }
  const uint32_t kept = __ballot_sync(0xffffffffu, lane < n_frames && has && frank < F);
  // ---- Top-K of the kept frames' blocks by counting rank
  int n_ok = 0;
#pragma unroll
  for (int r = 0; r < W; ++r) {
    if (wkey[r] != 0ull && !((kept >> wfr[r]) & 1u)) wkey[r] = 0ull;
    skeys[lane + 32 * r] = wkey[r];
    n_ok += __popc(__ballot_sync(0xffffffffu, wkey[r] != 0ull));
  }
  __syncwarp();
  const int take = min(a.k, n_ok);
  int rank[W];
#pragma unroll
  for (int r = 0; r < W; ++r) rank[r] = 0;
  const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(skeys);
#pragma unroll 4
  for (int f = 0; f < 16 * W; ++f) {
    const ulonglong2 v = k2[f];
#pragma unroll
    for (int r = 0; r < W; ++r) rank[r] += (v.x > wkey[r] ? 1 : 0) + (v.y > wkey[r] ? 1 : 0);
  }
#pragma unroll
  for (int r = 0; r < W; ++r)
    if (wkey[r] != 0ull && rank[r] < take) atomicOr(&bm[wid[r] >> 5], 1u << (wid[r] & 31));
#pragma unroll
  for (int r = 0; r < U; ++r) {
    const int m = mid[r];
    if (m >= NB || m < -1) report_status(a.status, PBSA_ERR_ARG);
    if (m >= 0 && m < NB && sel_len(a, bh, m) > 0) atomicOr(&bm[m >> 5], 1u << (m & 31));
  }
  __syncwarp();
  int total = 0;
  for (int w0 = 0; w0 < nbw; w0 += 32) {
    const uint32_t word = w0 + lane < nbw ? bm[w0 + lane] : 0u;
    int c = __popc(word);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
    total += c;
  }
  int32_t* out = a.idx + (bh * a.nQB_total + a.qb_offset + i) * static_cast<long>(a.Amax);
  int32_t* cnt = a.cnt + bh * a.nQB_total + a.qb_offset + i;
  if (total > a.Amax) {
    if (lane == 0) report_status(a.status, PBSA_ERR_SHAPE);
    for (int e = lane; e < a.Amax; e += 32) out[e] = -1;
    if (lane == 0) *cnt = 0;
    return;
  }
  int base = 0;
  for (int w0 = 0; w0 < nbw; w0 += 32) {
    uint32_t word = w0 + lane < nbw ? bm[w0 + lane] : 0u;
    const int c = __popc(word);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int pos = base + incl - c;
    while (word) {
      const int b = __ffs(word) - 1;
      out[pos++] = (w0 + lane) * 32 + b;
      word &= word - 1u;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  for (int e = total + lane; e < a.Amax; e += 32) out[e] = -1;
  if (lane == 0) *cnt = total;
}

}  // namespace dev
}  // namespace pbsa
