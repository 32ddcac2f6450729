// a4 + a5: local Top-K selection and list assembly, one warp per (b, h,
// query block).  The device code is in select_dev.cuh.
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "select_dev.cuh"

namespace pbsa {
namespace {

using namespace dev;

constexpr int kSelWarps = 4;

template <int W, int U>
__global__ void __launch_bounds__(32 * kSelWarps) select_kernel(SelArgs a) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x * kSelWarps + (threadIdx.x >> 5);
  if (i >= a.nQB) return;
  select_row<W, U>(a, i, blockIdx.y);
}

// The two-level (frame -> block) selection, one warp per (b, h, query block),
// each warp with its own slice of dynamic shared memory.
template <int W, int U>
__global__ void __launch_bounds__(32 * kSelWarps)
select_hier_kernel(SelArgs a, const int32_t* win_frame, int n_frames, int F) {
  extern __shared__ __align__(16) uint8_t smem[];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5;
  const int i = blockIdx.x * kSelWarps + warp;
  if (i >= a.nQB) return;
  select_row_hier<W, U>(a, win_frame, n_frames, F, i, blockIdx.y,
                        smem + warp * sel_hier_smem_per_warp<W>());
}

template <int W, int U>
cudaError_t launch_hier(const SelArgs& a, const int32_t* win_frame, int n_frames, int F,
                        dim3 grid, cudaStream_t st) {
  auto kern = select_hier_kernel<W, U>;
  const size_t smem = static_cast<size_t>(kSelWarps) * sel_hier_smem_per_warp<W>();
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    attr_set[dev] = true;
  }
  return launch(kern, grid, dim3(32 * kSelWarps), smem, st, a, win_frame, n_frames, F);
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
  cudaError_t err = cudaErrorInvalidValue;
  SelArgs a;
  a.scores = scores; a.win_ids = win_ids; a.mem_ids = mem_ids; a.blk_len = blk_len;
  a.blk_pos = blk_pos; a.idx = idx; a.cnt = cnt; a.status = status;
  a.nQB = nQB; a.NB = NB; a.n_win = n_win; a.k = k; a.n_mem = n_mem; a.mem_ld = mem_ld;
  a.mask = mask; a.q_pos0 = q_pos0; a.Tq = Tq; a.qc = d->q_chunk; a.bs = d->bs; a.Amax = Amax;
  a.qb_offset = qb_offset; a.nQB_total = nQB_total;
  a.slot_len = nullptr; a.slot_pos = nullptr; a.slot_ld = 0; a.n_slot = 0;
#define PBSA_SEL(WW, UU)                                                                       \
  if (W == WW && U == UU)                                                                      \
    err = launch(select_kernel<WW, UU>, grid, dim3(32 * kSelWarps), 0, st, a);
  PBSA_SEL(2, 2) PBSA_SEL(2, 4) PBSA_SEL(2, 8) PBSA_SEL(2, 16) PBSA_SEL(4, 2) PBSA_SEL(4, 4)
  PBSA_SEL(4, 8) PBSA_SEL(4, 16) PBSA_SEL(8, 2) PBSA_SEL(8, 4) PBSA_SEL(8, 8) PBSA_SEL(8, 16)
  PBSA_SEL(16, 2) PBSA_SEL(16, 4) PBSA_SEL(16, 8) PBSA_SEL(16, 16)
#undef PBSA_SEL
  if (err != cudaSuccess) PBSA_CHECK_LAUNCH("select_kernel");
  return PBSA_OK;
}

extern "C" int pbsa_select_hier(const pbsa_dims* d, const float* scores, int nQB, int NB,
                                const int32_t* win_ids, const int32_t* win_frame, int n_win,
                                int n_frames, int F, int k, const int32_t* mem_ids, int n_mem,
                                int mem_ld, const int32_t* blk_len, int mask, int q_pos0,
                                const int32_t* blk_pos, int Tq, int32_t* idx, int32_t* cnt,
                                int Amax, int qb_offset, int nQB_total, void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(scores && blk_len && idx && cnt, PBSA_ERR_ARG, "select_hier: NULL buffer");
  PBSA_CHECK_ARG(n_win >= 0 && n_win <= 32 * KPL, PBSA_ERR_SHAPE,
                 "select_hier: n_win must be in [0, 512]");
  PBSA_CHECK_ARG(n_win == 0 || (win_ids && win_frame), PBSA_ERR_ARG,
                 "select_hier: win_ids or win_frame is NULL");
  PBSA_CHECK_ARG(n_frames >= 1 && n_frames <= 32 && F >= 0, PBSA_ERR_SHAPE,
                 "select_hier: need 1 <= n_frames <= 32 and F >= 0");
  PBSA_CHECK_ARG(n_mem >= 0 && n_mem <= 32 * KPL && (n_mem == 0 || mem_ids), PBSA_ERR_ARG,
                 "select_hier: mem_ids is NULL or n_mem > 512");
  PBSA_CHECK_ARG(k >= 0 && nQB >= 1 && NB >= 1 && Amax >= 1, PBSA_ERR_SHAPE,
                 "select_hier: need k >= 0, nQB >= 1, NB >= 1, Amax >= 1");
  PBSA_CHECK_ARG(NB <= 32 * kSelBmWords, PBSA_ERR_SHAPE, "select_hier: NB must be <= 32768");
  const int take_max = k < n_win ? k : n_win;
  PBSA_CHECK_ARG(n_mem + take_max <= Amax, PBSA_ERR_SHAPE,
                 "select_hier: n_mem + min(k, n_win) must be <= Amax");
  PBSA_CHECK_ARG(mem_ld >= 0 && (mem_ld == 0 || mem_ld >= n_mem), PBSA_ERR_ARG,
                 "select_hier: mem_ld must be 0 or >= n_mem");
  if (mem_ld == 0) mem_ld = n_mem;
  PBSA_CHECK_ARG(mask == PBSA_MASK_CHUNK || (mask == PBSA_MASK_TOKEN && blk_pos), PBSA_ERR_ARG,
                 "select_hier: bad mask, or token mask without blk_pos");
  PBSA_CHECK_ARG(Tq >= 1 && qb_count(Tq, d->q_chunk, d->bs) == nQB, PBSA_ERR_SHAPE,
                 "select_hier: nQB must match the chunk tiling of Tq rows");
  PBSA_CHECK_ARG(qb_offset >= 0 && qb_offset + nQB <= nQB_total, PBSA_ERR_SHAPE,
                 "select_hier: qb_offset + nQB must be <= nQB_total");
  PBSA_CHECK_ARG(static_cast<long>(d->B) * d->H <= 65535, PBSA_ERR_SHAPE,
                 "select_hier: B*H must be <= 65535");
  int* status = device_status_ptr();
  PBSA_CHECK_ARG(status != nullptr, PBSA_ERR_CUDA, "select_hier: no device status word");
  dim3 grid((nQB + kSelWarps - 1) / kSelWarps, d->B * d->H);
  auto pick = [](int n) { return n <= 64 ? 2 : (n <= 128 ? 4 : (n <= 256 ? 8 : 16)); };
  const int W = pick(n_win), U = pick(n_mem);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaErrorInvalidValue;
  SelArgs a;
  a.scores = scores; a.win_ids = win_ids; a.mem_ids = mem_ids; a.blk_len = blk_len;
  a.blk_pos = blk_pos; a.idx = idx; a.cnt = cnt; a.status = status;
  a.nQB = nQB; a.NB = NB; a.n_win = n_win; a.k = k; a.n_mem = n_mem; a.mem_ld = mem_ld;
  a.mask = mask; a.q_pos0 = q_pos0; a.Tq = Tq; a.qc = d->q_chunk; a.bs = d->bs; a.Amax = Amax;
  a.qb_offset = qb_offset; a.nQB_total = nQB_total;
  a.slot_len = nullptr; a.slot_pos = nullptr; a.slot_ld = 0; a.n_slot = 0;
#define PBSA_HIER(WW, UU) \
  if (W == WW && U == UU) err = launch_hier<WW, UU>(a, win_frame, n_frames, F, grid, st);
  PBSA_HIER(2, 2) PBSA_HIER(2, 4) PBSA_HIER(2, 8) PBSA_HIER(2, 16) PBSA_HIER(4, 2)
  PBSA_HIER(4, 4) PBSA_HIER(4, 8) PBSA_HIER(4, 16) PBSA_HIER(8, 2) PBSA_HIER(8, 4)
  PBSA_HIER(8, 8) PBSA_HIER(8, 16) PBSA_HIER(16, 2) PBSA_HIER(16, 4) PBSA_HIER(16, 8)
  PBSA_HIER(16, 16)
#undef PBSA_HIER
  if (err != cudaSuccess) PBSA_CHECK_LAUNCH("select_hier_kernel");
  return PBSA_OK;
}
