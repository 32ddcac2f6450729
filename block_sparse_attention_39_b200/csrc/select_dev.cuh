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
};

// The attended list of query block i of head bh, computed by one warp.
template <int W, int U>
__device__ __forceinline__ void select_row(const SelArgs& a, int i, long bh) {
  const float* __restrict__ scores = a.scores;
  const int32_t* __restrict__ win_ids = a.win_ids;
  const int32_t* __restrict__ mem_ids = a.mem_ids;
  const int32_t* __restrict__ blk_len = a.blk_len;
  const int32_t* __restrict__ blk_pos = a.blk_pos;
  int32_t* __restrict__ idx = a.idx;
  int32_t* __restrict__ cnt = a.cnt;
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
  int wlen[W], wpos[W], mlen[U];
  float wsc[W];
#pragma unroll
  for (int r = 0; r < W; ++r) {
    const int j = wid[r];
    const bool in = j >= 0 && j < NB;
    if (r * 32 + lane < n_win && !in) report_status(status, PBSA_ERR_ARG);
    wlen[r] = in ? blk_len[bh * NB + j] : 0;
    wsc[r] = in ? srow[j] : 0.f;
    wpos[r] = (in && mask == PBSA_MASK_TOKEN) ? blk_pos[bh * NB + j] : 0;
  }
#pragma unroll
  for (int r = 0; r < U; ++r) {
    const int m = mid[r];
    // -1 names no block; any other id outside the pool is an argument error
    if (m >= NB || m < -1) report_status(status, PBSA_ERR_ARG);
    mlen[r] = (m >= 0 && m < NB) ? blk_len[bh * NB + m] : 0;
  }
  // ---- Top-K over the window (element order is irrelevant before the sort)
  uint64_t wkey[W];
  int n_ok = 0;
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
  const int take = min(k, n_ok);

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
  warp_bitonic_sort_desc<U>(key);

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
}

}  // namespace dev
}  // namespace pbsa
