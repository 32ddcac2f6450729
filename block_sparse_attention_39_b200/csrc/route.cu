// a1..a5 in one launch: the routing half of a decode step (pool + score ->
// memory update -> local selection) as one persistent, cooperative kernel.
//
// The four steps are the ones of pbsa_score_blocks, pbsa_update_memory and
// pbsa_select_local (same device code: pool_score_dev.cuh, update_dev.cuh,
// select_dev.cuh); what changes is the schedule.  A decode step's routing
// work is small (tens of MB of HBM traffic, a few thousand warps of sorting),
// so as separate kernels it is dominated by per-launch ramp-up and drain.  Here
// one CTA per SM slot (two per SM when they fit) walks every phase's items,
// and phases are separated by a grid barrier: an arrival counter in the
// caller's workspace, polled with a time limit, which the last CTA to leave
// resets to zero.  The launch is cooperative, so all CTAs are co-resident and
// the barrier cannot wait for a CTA that has not started.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <string>

#include "common.cuh"
#include "launch.h"
#include "pool_score_dev.cuh"
#include "select_dev.cuh"
#include "update_dev.cuh"

namespace pbsa {
namespace {

using namespace dev;

constexpr int kRouteThreads = 256;
constexpr size_t kRouteBarBytes = 256;   // workspace head: barrier words

struct RouteParams {
  PoolArgs pool;
  ScoreArgs score;
  UpdArgs upd;
  SelArgs sel;
  void* kpool;
  void* vpool;
  const void* stash;
  int32_t* blk_len;
  int32_t* blk_pos;
  float* k_bar;
  int32_t* slot_src;
  float* slot_w;
  unsigned long long* bar;   // [0] arrivals, [1] exits
  int do_update, n_score_items, n_jblk, n_itile, BH, P, n_rows, nQB;
  int* status;
  int64_t limit_ns;
};

// Grid-wide barrier number `k` (1, 2, ...): every CTA adds one arrival and
// waits until all G CTAs of barrier k have arrived.  Release/acquire through
// the CTA barrier plus a device-scope fence on either side of the counter.
__device__ __forceinline__ void grid_sync(const RouteParams& r, unsigned long long target) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(r.bar, 1ull);
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
      unsigned long long v;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(r.bar) : "memory");
      if (v >= target) break;
      if ((it & 63u) == 63u && static_cast<int64_t>(global_timer_ns() - t0) > r.limit_ns) {
        report_status(r.status, PBSA_ERR_TIMEOUT);
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
}

static_assert(kRouteScoreTile * kRouteScoreTile / 16 == kRouteThreads,
              "one 4 x 4 block of the score tile per routing thread");

template <typename T, int D, int W, int U>
__global__ void __launch_bounds__(kRouteThreads, 2) route_kernel(RouteParams r) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int cta = static_cast<int>(blockIdx.x), G = static_cast<int>(gridDim.x);
  unsigned long long target = 0;

  // a1: pooled means of the query blocks and of the listed key blocks
  pool_phase<T, D>(r.pool, cta, G, smem);
  grid_sync(r, target += G);

  // a2: scores and memory scores, one (b,h, 64 x 64 tile of S) item at a time
  for (int it = cta; it < r.n_score_items; it += G) {
    const int per_bh = r.n_jblk * r.n_itile, x = it % per_bh;
    score_item<D, kRouteScoreTile>(r.score, it / per_bh, x % r.n_jblk, x / r.n_jblk,
                                   reinterpret_cast<float*>(smem));
  }
  grid_sync(r, target += G);

  // a3: plan per (b,h), then stash (merge) and apply per (slot, b,h)
  if (r.do_update) {
    PlanSmem& ps = *reinterpret_cast<PlanSmem*>(smem);
    float* sk = reinterpret_cast<float*>(smem + ((sizeof(PlanSmem) + 15) / 16) * 16);
    for (int bh = cta; bh < r.BH; bh += G) plan_head(r.upd, bh, ps, sk);
    grid_sync(r, target += G);
    const int n_slot_items = r.P * r.BH;
    if (r.upd.policy == PBSA_MERGE_MEAN) {
      for (int it = cta; it < n_slot_items; it += G)
        stash_item<T>(r.upd, it % r.P, it / r.P, static_cast<const T*>(r.kpool),
                      static_cast<const T*>(r.vpool), static_cast<T*>(const_cast<void*>(r.stash)));
      grid_sync(r, target += G);
    }
    int* s_mref = reinterpret_cast<int*>(smem + 8 * D * sizeof(float));
    int* s_mlen = s_mref + kMaxItems;
    float* s_mw = reinterpret_cast<float*>(s_mlen + kMaxItems);
    for (int it = cta; it < n_slot_items; it += G)
      apply_item<T, D>(r.upd, it % r.P, it / r.P, static_cast<T*>(r.kpool),
                       static_cast<T*>(r.vpool), static_cast<const T*>(r.stash), r.blk_len,
                       r.blk_pos, r.k_bar, r.slot_src, r.slot_w,
                       reinterpret_cast<float(*)[D]>(smem), s_mref, s_mlen, s_mw);
    grid_sync(r, target += G);
  }

  // a4 + a5: one warp per (b,h, query block)
  {
    const int warp = threadIdx.x >> 5;
    constexpr int WPC = kRouteThreads / 32;
    for (int row = cta * WPC + warp; row < r.n_rows; row += G * WPC)
      select_row<W, U>(r.sel, row % r.nQB, row / r.nQB);
  }

  // leave the barrier words zeroed for the next call: the last CTA out resets
  // them (every other CTA has passed its last wait by then)
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned long long prev = atomicAdd(r.bar + 1, 1ull);
    if (prev == static_cast<unsigned long long>(G) - 1) {
      atomicExch(r.bar, 0ull);
      atomicExch(r.bar + 1, 0ull);
      __threadfence();
    }
  }
}

template <typename T, int D>
size_t route_smem(const RouteParams& r) {
  size_t m = pool_smem_bytes<T, D>(r.pool.stages, r.pool.bs);
  m = std::max(m, score_smem_bytes<D, kRouteScoreTile>());
  if (r.do_update) {
    size_t plan = (sizeof(PlanSmem) + 15) / 16 * 16;
    if (r.upd.policy == PBSA_MERGE_MEAN) plan += merge_key_smem(r.P, D);
    m = std::max(m, plan);
    m = std::max(m, static_cast<size_t>(8) * D * sizeof(float) + 3 * kMaxItems * sizeof(int));
  }
  return m;
}

// Cooperative launch of one instantiation; returns 1 when the shape does not
// fit a co-resident grid (the caller then runs the per-call kernels).
template <typename T, int D, int W, int U>
int launch_route(RouteParams& r, cudaStream_t s, int* rc) {
  auto kern = route_kernel<T, D, W, U>;
  const size_t smem = route_smem<T, D>(r);
  if (smem > 200 * 1024) return 1;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    attr_set[dev] = true;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRouteThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    return 1;
  const int G = std::min(per_sm, 2) * sm_count();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kRouteThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, r) != cudaSuccess) {
    *rc = PBSA_ERR_CUDA;
    set_error(std::string("route_kernel: ") + cudaGetErrorString(cudaGetLastError()));
  } else {
    *rc = PBSA_OK;
  }
  return 0;
}

template <typename T, int D>
int dispatch_route(int W, int U, RouteParams& r, cudaStream_t s, int* rc) {
  if (W == 2 && U == 2) return launch_route<T, D, 2, 2>(r, s, rc);
  if (W == 2 && U == 4) return launch_route<T, D, 2, 4>(r, s, rc);
  if (W == 4 && U == 2) return launch_route<T, D, 4, 2>(r, s, rc);
  if (W == 4 && U == 4) return launch_route<T, D, 4, 4>(r, s, rc);
  if (W == 8 && U == 2) return launch_route<T, D, 8, 2>(r, s, rc);
  if (W == 8 && U == 4) return launch_route<T, D, 8, 4>(r, s, rc);
  return 1;
}

}  // namespace
}  // namespace pbsa

extern "C" size_t pbsa_route_workspace(const pbsa_dims* d, int P, int n_cand) {
  if (d == nullptr || P < 0 || n_cand < 0 || d->B < 1 || d->H < 1) return 0;
  size_t upd = (P >= 1) ? pbsa_update_memory_workspace(d, P, n_cand) : 0;
  return pbsa::kRouteBarBytes + upd;
}

extern "C" int pbsa_route_step(const pbsa_dims* d, const pbsa_route_args* a, void* workspace,
                               size_t ws_bytes, void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(a != nullptr, PBSA_ERR_ARG, "route_step: args is NULL");
  PBSA_CHECK_ARG(a->Tq >= 1 && a->NB >= 1 && a->n_pool >= 0 && a->P >= 0 && a->n_cand >= 0,
                 PBSA_ERR_SHAPE, "route_step: need Tq >= 1, NB >= 1, n_pool, P, n_cand >= 0");
  const size_t need = pbsa_route_workspace(d, a->P, a->n_cand);
  PBSA_CHECK_ARG(workspace != nullptr && ws_bytes >= need && aligned(workspace, 256),
                 PBSA_ERR_WORKSPACE,
                 "route_step: workspace missing, too small or not 256-byte aligned (need " +
                     std::to_string(need) + " bytes)");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  void* upd_ws = ws + kRouteBarBytes;
  const size_t upd_bytes = ws_bytes - kRouteBarBytes;
  const bool do_update = a->P >= 1 && a->n_cand >= 1;
  const int nQB = qb_count(a->Tq, d->q_chunk, d->bs);
  const int take_max = a->k < a->n_win ? a->k : a->n_win;
  auto pick = [](int n) { return n <= 64 ? 2 : (n <= 128 ? 4 : (n <= 256 ? 8 : 16)); };
  const int W = pick(a->n_win), U = pick(a->n_mem + take_max);

  // the per-call path: the three entry points in order (they validate their
  // own arguments); used when the fused kernel has no instantiation or no
  // co-resident grid for this shape
  auto per_call = [&]() -> int {
    int r = pbsa_score_blocks(d, a->q, a->Tq, a->kpool, a->NB, a->blk_len, a->pool_ids,
                              a->n_pool, a->q_bar, a->k_bar, a->scores, a->mem_score, stream);
    if (r) return r;
    if (do_update) {
      r = pbsa_update_memory(d, a->kpool, a->vpool, a->NB, a->blk_len, a->blk_pos, a->k_bar,
                             a->P, a->n_sink, a->slot_src, a->slot_w, a->cand_ids, a->cand_src,
                             a->n_cand, a->mem_score, a->policy, upd_ws, upd_bytes, stream);
      if (r) return r;
    }
    return pbsa_select_local(d, a->scores, nQB, a->NB, a->win_ids, a->n_win, a->k, a->mem_ids,
                             a->n_mem, 0, a->blk_len, a->mask, a->q_pos0, a->blk_pos, a->Tq,
                             a->idx, a->cnt, a->Amax, 0, nQB, stream);
  };

  // ---- the fused kernel's own argument checks (the union of the three calls')
  PBSA_CHECK_ARG(a->q && a->kpool && a->blk_len && a->q_bar && a->k_bar && a->scores &&
                     a->mem_score && a->idx && a->cnt,
                 PBSA_ERR_ARG, "route_step: NULL buffer");
  PBSA_CHECK_ARG(a->n_pool == 0 || a->pool_ids, PBSA_ERR_ARG, "route_step: pool_ids is NULL");
  PBSA_CHECK_ARG(aligned(a->q, 16) && aligned(a->kpool, 16) && aligned(a->q_bar, 16) &&
                     aligned(a->k_bar, 16) && aligned(a->scores, 4) && aligned(a->mem_score, 4),
                 PBSA_ERR_ALIGN, "route_step: misaligned buffer");
  PBSA_CHECK_ARG(static_cast<long>(d->B) * d->H <= 65535, PBSA_ERR_SHAPE,
                 "route_step: B*H must be <= 65535");
  PBSA_CHECK_ARG(a->n_win >= 0 && a->n_win <= 512 && (a->n_win == 0 || a->win_ids),
                 PBSA_ERR_SHAPE, "route_step: n_win must be in [0, 512] with win_ids");
  PBSA_CHECK_ARG(a->n_mem >= 0 && (a->n_mem == 0 || a->mem_ids), PBSA_ERR_ARG,
                 "route_step: mem_ids is NULL");
  PBSA_CHECK_ARG(a->k >= 0 && a->Amax >= 1 && a->n_mem + take_max <= a->Amax &&
                     a->n_mem + take_max <= 512,
                 PBSA_ERR_SHAPE, "route_step: n_mem + min(k, n_win) must be <= min(Amax, 512)");
  PBSA_CHECK_ARG(a->mask == PBSA_MASK_CHUNK || (a->mask == PBSA_MASK_TOKEN && a->blk_pos),
                 PBSA_ERR_ARG, "route_step: bad mask, or token mask without blk_pos");
  if (do_update) {
    PBSA_CHECK_ARG(a->vpool && a->blk_pos && a->slot_src && a->slot_w && a->cand_ids &&
                       a->cand_src && aligned(a->vpool, 16),
                   PBSA_ERR_ARG, "route_step: NULL or misaligned update buffer");
    PBSA_CHECK_ARG(a->P <= 256 && a->NB >= a->P && a->n_sink >= 0 && a->n_sink <= a->P &&
                       (a->P - a->n_sink) + a->n_cand <= 256,
                   PBSA_ERR_SHAPE, "route_step: need P <= 256, NB >= P, (P - n_sink) + n_cand <= 256");
    PBSA_CHECK_ARG(a->policy == PBSA_EVICT || a->policy == PBSA_MERGE_MEAN, PBSA_ERR_ARG,
                   "route_step: bad policy");
  }
  const long n_items = static_cast<long>(d->B) * d->H * (nQB + a->n_pool);
  PBSA_CHECK_ARG(n_items < (1L << 31), PBSA_ERR_SHAPE, "route_step: too many blocks to pool");
  const long n_score_items = static_cast<long>(d->B) * d->H *
                             ((a->NB + kRouteScoreTile - 1) / kRouteScoreTile) *
                             ((nQB + kRouteScoreTile - 1) / kRouteScoreTile);
  PBSA_CHECK_ARG(n_score_items < (1L << 31), PBSA_ERR_SHAPE, "route_step: too many score tiles");
  int* status = device_status_ptr();
  PBSA_CHECK_ARG(status != nullptr, PBSA_ERR_CUDA, "route_step: no device status word");

  RouteParams r;
  const int BH = d->B * d->H;
  r.pool.q = a->q; r.pool.kpool = a->kpool; r.pool.blk_len = a->blk_len;
  r.pool.pool_ids = a->pool_ids; r.pool.q_bar = a->q_bar; r.pool.k_bar = a->k_bar;
  r.pool.Tq = a->Tq; r.pool.qc = d->q_chunk; r.pool.NB = a->NB; r.pool.bs = d->bs;
  r.pool.nQB = nQB; r.pool.n_pool = a->n_pool; r.pool.n_items = static_cast<int>(n_items);
  r.pool.status = status; r.pool.limit_ns = wait_limit_ns();
  r.pool.stages = d->dtype == PBSA_BF16
                      ? (d->D == 128 ? pool_stages<__nv_bfloat16, 128>(d->bs)
                                     : pool_stages<__nv_bfloat16, 64>(d->bs))
                      : (d->D == 128 ? pool_stages<float, 128>(d->bs) : pool_stages<float, 64>(d->bs));
  const int qc = d->q_chunk > 0 ? d->q_chunk : a->Tq;
  r.score.q_bar = a->q_bar; r.score.k_bar = a->k_bar; r.score.scores = a->scores;
  r.score.mem = a->mem_score; r.score.nQB = nQB; r.score.NB = a->NB;
  r.score.per_group = (qc + d->bs - 1) / d->bs; r.score.groups = (a->Tq + qc - 1) / qc;
  r.score.scale = d->scale;
  r.upd.B = d->B; r.upd.H = d->H; r.upd.D = d->D; r.upd.bs = d->bs; r.upd.NB = a->NB;
  r.upd.P = a->P; r.upd.n_sink = a->n_sink; r.upd.n_cand = a->n_cand; r.upd.policy = a->policy;
  r.upd.M = a->P + a->n_cand; r.upd.blk_len = a->blk_len; r.upd.blk_pos = a->blk_pos;
  r.upd.k_bar = a->k_bar; r.upd.slot_src = a->slot_src; r.upd.slot_w = a->slot_w;
  r.upd.cand_ids = a->cand_ids; r.upd.cand_src = a->cand_src; r.upd.mem = a->mem_score;
  r.upd.ws = upd_ws; r.upd.status = status;
  r.sel.scores = a->scores; r.sel.win_ids = a->win_ids; r.sel.mem_ids = a->mem_ids;
  r.sel.blk_len = a->blk_len; r.sel.blk_pos = a->blk_pos; r.sel.idx = a->idx; r.sel.cnt = a->cnt;
  r.sel.status = status; r.sel.nQB = nQB; r.sel.NB = a->NB; r.sel.n_win = a->n_win;
  r.sel.k = a->k; r.sel.n_mem = a->n_mem; r.sel.mem_ld = a->n_mem; r.sel.mask = a->mask;
  r.sel.q_pos0 = a->q_pos0; r.sel.Tq = a->Tq; r.sel.qc = d->q_chunk; r.sel.bs = d->bs;
  r.sel.Amax = a->Amax; r.sel.qb_offset = 0; r.sel.nQB_total = nQB;
  r.kpool = a->kpool; r.vpool = a->vpool;
  r.stash = do_update ? static_cast<const char*>(upd_ws) +
                            static_cast<size_t>(BH) * dev::plan_bytes(a->P, a->P + a->n_cand)
                      : nullptr;
  r.blk_len = a->blk_len; r.blk_pos = a->blk_pos; r.k_bar = a->k_bar;
  r.slot_src = a->slot_src; r.slot_w = a->slot_w;
  r.bar = reinterpret_cast<unsigned long long*>(ws);
  r.do_update = do_update ? 1 : 0;
  r.n_jblk = (a->NB + kRouteScoreTile - 1) / kRouteScoreTile;
  r.n_itile = (nQB + kRouteScoreTile - 1) / kRouteScoreTile;
  r.n_score_items = BH * r.n_jblk * r.n_itile;
  r.BH = BH; r.P = a->P; r.n_rows = BH * nQB; r.nQB = nQB;
  r.status = status; r.limit_ns = wait_limit_ns();

  int launched_rc = PBSA_OK;
  int fallback = 1;
  if (d->dtype == PBSA_BF16)
    fallback = d->D == 128 ? dispatch_route<__nv_bfloat16, 128>(W, U, r, s, &launched_rc)
                           : dispatch_route<__nv_bfloat16, 64>(W, U, r, s, &launched_rc);
  else
    fallback = d->D == 128 ? dispatch_route<float, 128>(W, U, r, s, &launched_rc)
                           : dispatch_route<float, 64>(W, U, r, s, &launched_rc);
  if (fallback) return per_call();
  return launched_rc;
}
