// a4 + a5: local Top-K selection inside the sliding window and assembly of the
// attended-block list (persistent memory united with the local selection).
//
// Sparse Forcing restricts attention inside the recent window to the Top-K
// blocks most relevant to each query (gist.science/es, section 2
// "Arquitectura Propuesta", item "Ventana Local") and attends the persistent
// memory densely (PBSA item "Atención Híbrida").
//
// One warp per (b, h, query block): the window's scores become 64-bit keys
// (orderable score, ~id), a warp-wide bitonic sort over 256 keys held in
// registers (up to 512 keys) picks the Top-K, and a second bitonic sort merges
// the selection with the memory ids into an ascending, duplicate-free list.
#include <cuda_runtime.h>

#include "common.cuh"

namespace pbsa {
namespace {

constexpr int KPL = 16;                 // capacity: 512 keys per warp
constexpr int kSelWarps = 4;

// W: keys per lane of the window sort; U: keys per lane of the union sort
// (32*W >= n_win, 32*U >= n_mem + min(k, n_win)); both <= KPL.
template <int W, int U>
__global__ void __launch_bounds__(32 * kSelWarps)
select_kernel(const float* __restrict__ scores, int nQB, int NB, const int32_t* __restrict__ win_ids,
              int n_win, int k, const int32_t* __restrict__ mem_ids, int n_mem, int mem_ld,
              const int32_t* __restrict__ blk_len, int mask, int q_pos0,
              const int32_t* __restrict__ blk_pos, int Tq, int qc, int bs, int32_t* __restrict__ idx,
              int32_t* __restrict__ cnt, int Amax, int qb_offset, int nQB_total, int* status) {
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * kSelWarps + (threadIdx.x >> 5);
  if (i >= nQB) return;
  const long bh = blockIdx.y;
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
    if (lane == 0) report_status(status, PBSA_ERR_SHAPE);
    return;
  }
#pragma unroll
  for (int r = 0; r < U; ++r) {
    if (keep[r]) out[pos++] = static_cast<int32_t>(0xffffffffu - static_cast<uint32_t>(key[r]));
  }
  for (int e = total + lane; e < Amax; e += 32) out[e] = -1;
  if (lane == 0) cnt[bh * nQB_total + qb_offset + i] = total;
}

}  // namespace
}  // namespace pbsa

extern "C" int pbsa_select_local(const pbsa_dims* d, const float* scores, int nQB, int NB,
                                 const int32_t* win_ids, int n_win, int k, const int32_t* mem_ids,
                                 int n_mem, int mem_ld, const int32_t* blk_len, int mask, int q_pos0,
                                 const int32_t* blk_pos, int Tq, int32_t* idx, int32_t* cnt,
                                 int Amax, int qb_offset, int nQB_total, void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(scores && blk_len && idx && cnt, PBSA_ERR_ARG, "select_local: NULL buffer");
  PBSA_CHECK_ARG(n_win >= 0 && n_win <= 32 * KPL, PBSA_ERR_SHAPE,
                 "select_local: n_win must be in [0, 512]");
  PBSA_CHECK_ARG(n_win == 0 || win_ids, PBSA_ERR_ARG, "select_local: win_ids is NULL");
  PBSA_CHECK_ARG(n_mem >= 0 && (n_mem == 0 || mem_ids), PBSA_ERR_ARG,
                 "select_local: mem_ids is NULL");
  PBSA_CHECK_ARG(k >= 0 && nQB >= 1 && NB >= 1 && Amax >= 1, PBSA_ERR_SHAPE,
                 "select_local: need k >= 0, nQB >= 1, NB >= 1, Amax >= 1");
  const int take_max = k < n_win ? k : n_win;
  PBSA_CHECK_ARG(n_mem + take_max <= Amax && n_mem + take_max <= 32 * KPL, PBSA_ERR_SHAPE,
                 "select_local: n_mem + min(k, n_win) must be <= min(Amax, 512)");
  PBSA_CHECK_ARG(mem_ld >= 0 && (mem_ld == 0 || mem_ld >= n_mem), PBSA_ERR_ARG,
                 "select_local: mem_ld must be 0 or >= n_mem");
  if (mem_ld == 0) mem_ld = n_mem;
  PBSA_CHECK_ARG(mask == PBSA_MASK_CHUNK || mask == PBSA_MASK_TOKEN, PBSA_ERR_ARG,
                 "select_local: bad mask");
  PBSA_CHECK_ARG(mask == PBSA_MASK_CHUNK || blk_pos, PBSA_ERR_ARG,
                 "select_local: token mask needs blk_pos");
  PBSA_CHECK_ARG(Tq >= 1 && qb_count(Tq, d->q_chunk, d->bs) == nQB, PBSA_ERR_SHAPE,
                 "select_local: nQB must match the chunk tiling of Tq rows");
  PBSA_CHECK_ARG(qb_offset >= 0 && qb_offset + nQB <= nQB_total, PBSA_ERR_SHAPE,
                 "select_local: qb_offset + nQB must be <= nQB_total");
  PBSA_CHECK_ARG(static_cast<long>(d->B) * d->H <= 65535, PBSA_ERR_SHAPE,
                 "select_local: B*H must be <= 65535");
  int* status = device_status_ptr();
  PBSA_CHECK_ARG(status != nullptr, PBSA_ERR_CUDA, "select_local: no device status word");
  dim3 grid((nQB + kSelWarps - 1) / kSelWarps, d->B * d->H);
  auto pick = [](int n) { return n <= 64 ? 2 : (n <= 128 ? 4 : (n <= 256 ? 8 : 16)); };
  const int W = pick(n_win), U = pick(n_mem + take_max);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
#define PBSA_SEL(WW, UU)                                                                       \
  if (W == WW && U == UU)                                                                      \
    select_kernel<WW, UU><<<grid, 32 * kSelWarps, 0, st>>>(                                    \
        scores, nQB, NB, win_ids, n_win, k, mem_ids, n_mem, mem_ld, blk_len, mask, q_pos0,      \
        blk_pos, Tq,                                                                           \
        d->q_chunk, d->bs, idx, cnt, Amax, qb_offset, nQB_total, status);
  PBSA_SEL(2, 2) PBSA_SEL(2, 4) PBSA_SEL(2, 8) PBSA_SEL(2, 16) PBSA_SEL(4, 2) PBSA_SEL(4, 4)
  PBSA_SEL(4, 8) PBSA_SEL(4, 16) PBSA_SEL(8, 2) PBSA_SEL(8, 4) PBSA_SEL(8, 8) PBSA_SEL(8, 16)
  PBSA_SEL(16, 2) PBSA_SEL(16, 4) PBSA_SEL(16, 8) PBSA_SEL(16, 16)
#undef PBSA_SEL
  PBSA_CHECK_LAUNCH("select_kernel");
  return PBSA_OK;
}
