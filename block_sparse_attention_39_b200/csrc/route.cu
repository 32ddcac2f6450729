// a1..a5 in one launch: the routing half of a decode step (pool + score ->
// memory update -> local selection) as one persistent, dependency-driven
// kernel.
//
// The four steps are the ones of pbsa_score_blocks, pbsa_update_memory and
// pbsa_select_local (same device code: pool_score_dev.cuh, update_dev.cuh,
// select_dev.cuh); what changes is the schedule.  A decode step's routing
// work is small (tens of MB of HBM traffic, a few thousand warps of sorting),
// so as separate kernels it is dominated by per-launch ramp-up and drain, and
// with grid-wide barriers between the steps every step waits for the slowest
// head of the step before it.
//
// Here every piece of work is a numbered ticket, handed out in order by one
// atomic counter, and each ticket waits only for the tickets it reads.  In
// ticket order:
//
//   pool    (b,h, block)    a block's pooled mean (queries, then listed keys)
//   plan    (b,h)           the memory update's plan; waits for every pool
//                           ticket of its head and computes the memory scores
//                           of its candidates itself, with the arithmetic of
//                           the score tiles (so the same bits)
//   score   (b,h, tile)     a 32 x 32 tile of S and its memory scores; waits
//                           for every pool ticket of its head
//   stash   (b,h, slot)     merge policy only; waits for the head's plan
//   select  (b,h, 8 rows)   eight attended lists, one per warp; waits for the
//                           head's score tiles and plan (the plan states the
//                           slots' lengths after the update, so the lists do
//                           not wait for the slot copies)
//   apply   (b,h, slot)     writes one slot; waits for the plan, for the
//                           head's score tiles (they read the slots' pooled
//                           keys from before the update) and, under the merge
//                           policy, for the head's stash tickets
//
// The update plan is the longest chain, so its tickets come first after
// the pooling.
// Tickets are numbered so that every dependency has a lower number, and a CTA
// only waits for a ticket after claiming its own, so the ticket it waits for
// is held by a CTA that is already running: the waits always end, whatever
// the number of co-resident CTAs.  Completion is counted per (b,h) in the
// caller's workspace (release: CTA barrier, then one thread's device-scope
// fence and atomic add; acquire: one thread's ld.acquire.gpu, then a CTA
// barrier).  Every wait is bounded; a wait that runs out sets the status word
// and a kernel-wide abort flag, after which the remaining tickets are claimed
// and skipped.  The last CTA to leave resets the counters to zero.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <string>

#include "common.cuh"
#include "launch.h"

#ifdef PBSA_ROUTE_TRACE
namespace pbsa {
__device__ unsigned long long g_plan_trace[64][8];
}
namespace pbsa {
__device__ unsigned long long g_sel_trace[12][48][8];
}
#define SEL_TRACE(i, bh, k)                                                        \
  do {                                                                           \
    if ((threadIdx.x & 31) == 0 && (bh) < 12 && (i) < 48) {                      \
      unsigned long long t_;                                                     \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                     \
      ::pbsa::g_sel_trace[(bh)][(i)][(k)] = t_;                                  \
    }                                                                            \
  } while (0)
#define PLAN_TRACE(bh, k)                                                          \
  do {                                                                           \
    if (threadIdx.x == 0 && (bh) < 64) {                                         \
      unsigned long long t_;                                                     \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                     \
      ::pbsa::g_plan_trace[(bh)][(k)] = t_;                                      \
    }                                                                            \
  } while (0)
#endif

#include "pool_score_dev.cuh"
#include "select_dev.cuh"
#include "update_dev.cuh"

namespace pbsa {
namespace {

using namespace dev;

constexpr int kRouteThreads = 256;
constexpr int kRouteSelRows = kRouteThreads / 32;    // rows per select ticket (one per warp)
constexpr int kCtlWords = 4;                         // ticket, exits, abort, spare

// Bytes of the counter area at the head of the workspace: the control words
// and five per-(b,h) completion counters.
inline size_t route_ctl_bytes(long BH) { return align_up((kCtlWords + 5 * BH) * 4, 256); }

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
  unsigned* ctl;          // [0] next ticket, [1] CTAs finished, [2] abort flag
  unsigned* pool_done;    // [BH] each: completion counter of one kind of ticket
  unsigned* score_done;
  unsigned* plan_done;
  unsigned* stash_done;
  unsigned* apply_done;
  int n_ctl_words;        // words to reset: kCtlWords + 5 * BH
  int BH, P, nQB, n_jblk, n_itile;
  int per_pool;           // pool tickets per head
  int per_score;          // score tiles per head
  int per_sel;            // select tickets per head
  int merge;              // stash tickets exist
  // first ticket of each kind, in ticket order (pool tickets start at 0);
  // t_end is the number of tickets
  int t_plan, t_score, t_stash, t_sel, t_apply, t_end;
  int* status;
  int64_t limit_ns;
  int debug;              // test hook: bit 1 withholds head 0's pool completions
};

// Per-ticket time stamps for schedule studies, compiled in only with
// -DPBSA_ROUTE_TRACE (the library built without it records nothing).
#ifdef PBSA_ROUTE_TRACE
__device__ unsigned long long g_route_trace[1 << 15][4];
__device__ unsigned long long g_route_cta[1024][4];
#define ROUTE_TRACE(tk, slot)                                                      \
  do {                                                                           \
    if (threadIdx.x == 0 && (tk) >= 0 && (tk) < (1 << 15))                        \
      g_route_trace[(tk)][(slot)] = global_timer_ns();                           \
  } while (0)
#define ROUTE_TRACE_CTA(slot)                                                      \
  do {                                                                           \
    if (threadIdx.x == 0 && blockIdx.x < 1024) g_route_cta[blockIdx.x][(slot)] = global_timer_ns(); \
  } while (0)
#else
#define ROUTE_TRACE(tk, slot) do {} while (0)
#define ROUTE_TRACE_CTA(slot) do {} while (0)
#endif

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_relaxed(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ int claim(const RouteParams& r) {
  return static_cast<int>(atomicAdd(r.ctl, 1u));
}

// Marks one ticket done: every thread's writes of the ticket precede the CTA
// barrier, which precedes thread 0's device-scope fence and the count.
__device__ __forceinline__ void signal_done(unsigned* ctr) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
  }
}

// Waits until *ctr >= target (thread 0 polls; the CTA barrier then orders every
// thread's reads after the acquiring load).  Returns false after the kernel
// aborted or when the time limit runs out (which aborts the kernel).
__device__ bool wait_count(const RouteParams& r, const unsigned* ctr, unsigned target) {
  bool ok = true;
  if (threadIdx.x == 0) {
    ok = ld_relaxed(r.ctl + 2) == 0;
    if (ok && ld_acquire(ctr) < target) {
      const uint64_t t0 = global_timer_ns();
      for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if (ld_acquire(ctr) >= target) break;
        if ((it & 15u) == 0) {
          if (ld_relaxed(r.ctl + 2) != 0) { ok = false; break; }
          if (static_cast<int64_t>(global_timer_ns() - t0) > r.limit_ns) {
            report_status(r.status, PBSA_ERR_TIMEOUT);
            atomicExch(r.ctl + 2, 1u);
            ok = false;
            break;
          }
        }
      }
    }
  }
  // the barrier carries thread 0's answer to every thread
  return __syncthreads_and(ok ? 1 : 0) != 0;
}

// ------------------------------------------------------------------ pooling
// Counts pool ticket tk done (its mean was written before the caller's last
// CTA barrier).  Debug bit 1 (pbsa_set_debug) withholds the counts of head 0,
// so that head's dependent tickets time out: the failure path under test.
__device__ __forceinline__ void pool_signal(const RouteParams& r, int tk) {
  const int bh = tk / r.per_pool;
  if ((r.debug & 2) && bh == 0) return;
  __threadfence();
  atomicAdd(r.pool_done + bh, 1u);
  ROUTE_TRACE(tk, 2);
}

// The pool tickets, claimed one at a time by thread 0 and streamed through a
// ring of shared-memory stages (untiled bulk copies completing on mbarriers,
// the same summation as pool_phase, so the means are bit-identical).  Returns
// the first ticket this CTA claimed past the pool range, or -1 if the CTA
// aborted before claiming one.
template <typename T, int D>
__device__ __forceinline__ int route_pool(const RouteParams& r, uint8_t* smem) {
  const PoolArgs& a = r.pool;
  constexpr int ROW = D * static_cast<int>(sizeof(T));
  const int S = a.stages;
  const int stage_bytes = a.bs * ROW;
  float* red = reinterpret_cast<float*>(smem + S * stage_bytes);       // [2][8][D]
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 2 * 8 * D);        // [S]
  long* s_out = reinterpret_cast<long*>(bars + S);                      // [S]
  int* s_n = reinterpret_cast<int*>(s_out + S);                         // [S]
  int* s_tk = s_n + S;                                                  // [S] its ticket
  int* s_ctl = s_tk + S;            // [0] items issued, [1] first ticket past the pool range
  volatile int* abort_flag = s_ctl + 2;
  const int t = threadIdx.x;
  const int n_pool_items = r.t_plan;

  // thread 0: claim a ticket; a pool ticket is issued into stage k % S
  auto issue = [&](int k) -> bool {
    const int tk = claim(r);
    if (tk >= n_pool_items) {
      ROUTE_TRACE(tk, 0);
      s_ctl[1] = tk;
      return false;
    }
    const int s = k % S;
    const T* src;
    long out;
    int n;
    ROUTE_TRACE(tk, 0);
    pool_item<T, D>(a, tk, src, out, n);
    ROUTE_TRACE(tk, 1);
    s_n[s] = n;
    s_out[s] = out;
    s_tk[s] = tk;
    const uint32_t bar = smem_u32(&bars[s]);
    if (n > 0) {
      mbar_expect_tx(bar, static_cast<uint32_t>(n * ROW));
      bulk_load(smem_u32(smem + s * stage_bytes), src, static_cast<uint32_t>(n * ROW), bar);
    } else {
      mbar_arrive(bar);
    }
    s_ctl[0] = k + 1;
    return true;
  };

  if (t == 0) {
    for (int s = 0; s < S; ++s) mbar_init(smem_u32(&bars[s]), 1);
    *abort_flag = 0;
    s_ctl[0] = 0;
    s_ctl[1] = -1;
    fence_mbar_init();
    for (int k = 0; k < S; ++k)
      if (!issue(k)) break;
  }
  bool ok = true;
  int prev_tk = -1;
  int k = 0;
  for (;; ++k) {
    // thread 0 alone knows how many tickets it has issued
    if (!__syncthreads_or(t == 0 && k < s_ctl[0])) break;
    // the previous item's mean was written before this barrier
    if (t == 0 && k > 0) pool_signal(r, prev_tk);
    const int s = k % S;
    ok = mbar_wait(smem_u32(&bars[s]), static_cast<uint32_t>((k / S) & 1), abort_flag, a.status,
                   a.limit_ns);
    if (__syncthreads_or(!ok)) { ok = false; break; }
    const int n = s_n[s];
    const long oo = s_out[s];
    prev_tk = s_tk[s];
    float* rb = red + (k & 1) * 8 * D;
    row_sums<T, D>(smem + s * stage_bytes, n, rb);
    __syncthreads();   // stage s fully read; partial sums of item k complete
    if (t == 0 && s_ctl[1] < 0) issue(k + S);
    if (t < D && oo != -1) {
      float* o = oo >= 0 ? a.q_bar + oo : a.k_bar + (-(oo + 2));
      o[t] = row_mean<D>(rb, n);
    }
  }
  if (ok) {
    if (t == 0 && k > 0) pool_signal(r, prev_tk);
  } else if (t == 0) {
    atomicExch(r.ctl + 2, 1u);
    // no copy may still be in flight when the stages are reused
    const int issued = s_ctl[0];
    for (int j = max(0, issued - S); j < issued; ++j)
      mbar_drain(smem_u32(&bars[j % S]), static_cast<uint32_t>((j / S) & 1), a.status, a.limit_ns);
  }
  __syncthreads();
  const int first = s_ctl[1];
  if (t < S) mbar_inval(smem_u32(&bars[t]));
  __syncthreads();
  return first;
}

// ------------------------------------------------------------ other tickets
// Memory scores of head bh's plan items (its occupied non-sink slots, then the
// candidates, in plan_head's item order) into item_mem: the mean of the
// head's pooled queries (group 0; the update needs a single query chunk),
// summed in block order and divided once, then scale * quad_dot with each
// item's pooled key -- the computation of score_item, so each value has the
// bits of the memory score a score tile writes for that block.  Rows are
// staged in shared memory by 16-byte asynchronous copies: the query rows
// (kPlanQRows at a time, into XQ) go out at once, the items' pooled keys
// (kPlanKRows at a time, into XK) as soon as the items' block ids are read,
// so a decode step's prologue costs about two round trips to memory.
constexpr int kPlanQRows = 40, kPlanKRows = 136;

// Shared-memory layout of a plan ticket: XQ (later the plan's own PlanSmem),
// item ids, the query mean, the items' memory scores, XK (later the kept
// slots' pooled keys of a merge).
template <int D>
struct PlanLayout {
  static constexpr size_t kXQ = ((sizeof(PlanSmem) > kPlanQRows * D * 4 ? sizeof(PlanSmem)
                                                                          : kPlanQRows * D * 4) +
                                 15) / 16 * 16;
  static constexpr size_t kPhys = kXQ;
  static constexpr size_t kQm = kPhys + kMaxItems * 4;
  static constexpr size_t kMem = kQm + D * 4;
  static constexpr size_t kXK = kMem + kMaxItems * 4;
  static size_t bytes(int P, int policy) {
    const size_t xk = static_cast<size_t>(kPlanKRows) * score_pitch<D>() * 4;
    const size_t sk = policy == PBSA_MERGE_MEAN ? merge_key_smem(P, D) : 0;
    return kXK + (xk > sk ? xk : sk);
  }
};

// rows[i] (or row i if rows is NULL) of a [*, D] fp32 matrix into row i of
// dst (row pitch `pitch` floats), as one group of asynchronous copies
template <int D>
__device__ __forceinline__ void stage_rows(float* dst, int pitch, const float* base,
                                           const int* rows, int n) {
  for (int e = threadIdx.x; e < n * (D / 4); e += kRouteThreads) {
    const int row = e / (D / 4), c4 = e % (D / 4);
    const int src_row = rows ? rows[row] : row;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst + row * pitch + c4 * 4)),
                 "l"(base + static_cast<long>(src_row) * D + c4 * 4)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

template <int D>
__device__ void plan_item_mem(const RouteParams& r, long bh, uint8_t* smem) {
  using L = PlanLayout<D>;
  constexpr int PT = score_pitch<D>();
  float* XQ = reinterpret_cast<float*>(smem);
  int* item_phys = reinterpret_cast<int*>(smem + L::kPhys);
  float* qm = reinterpret_cast<float*>(smem + L::kQm);
  float* item_mem = reinterpret_cast<float*>(smem + L::kMem);
  float* XK = reinterpret_cast<float*>(smem + L::kXK);
  const int t = threadIdx.x;
  const UpdArgs& a = r.upd;
  const int n_dyn = a.P - a.n_sink, NI = n_dyn + a.n_cand;
  const int n_rows = min(r.score.nQB, r.score.per_group);
  const float* qrows = r.score.q_bar + bh * r.score.nQB * D;
  const float* krows = a.k_bar + bh * a.NB * static_cast<long>(D);
  __syncthreads();                        // shared memory of the previous ticket
  stage_rows<D>(XQ, D, qrows, nullptr, min(kPlanQRows, n_rows));
  if (t < NI) {
    int phys = 0;                         // an invalid item reads block 0; its score is unused
    if (t < n_dyn) {
      const int s = a.n_sink + t;
      if (a.slot_src[bh * a.P + s] >= 0) phys = s;
    } else {
      const int c = a.cand_ids[t - n_dyn];
      if (c >= 0 && c < a.NB) phys = c;
    }
    item_phys[t] = phys;
  }
  __syncthreads();                        // item_phys complete
  stage_rows<D>(XK, PT, krows, item_phys, min(kPlanKRows, NI));
  // the query mean, kPlanQRows rows at a time, summed in block order
  float sum = 0.f;
  for (int r0 = 0; r0 < n_rows; r0 += kPlanQRows) {
    const int nr = min(kPlanQRows, n_rows - r0);
    if (r0 > 0) {
      __syncthreads();                    // XQ read
      stage_rows<D>(XQ, D, qrows + static_cast<long>(r0) * D, nullptr, nr);
      asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 1;\n" ::: "memory");   // the query rows
    }
    __syncthreads();
    if (t < D) {
#pragma unroll 8
      for (int i = 0; i < nr; ++i) sum += XQ[i * D + t];
    }
  }
  if (t < D) qm[t] = sum / static_cast<float>(n_rows);
  const int p = t & 3;
  for (int u0 = 0; u0 < NI; u0 += kPlanKRows) {
    const int nu = min(kPlanKRows, NI - u0);
    if (u0 > 0) {
      __syncthreads();                    // XK read
      stage_rows<D>(XK, PT, krows, item_phys + u0, nu);
    }
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();                      // also publishes qm
    // one row per quad; every lane of a warp takes part in the shuffles
    for (int u = t >> 2; u < (nu + 63) / 64 * 64; u += kRouteThreads / 4) {
      const float sdot = quad_dot<D>(qm, XK + min(u, nu - 1) * PT, p);
      if (p == 0 && u < nu) item_mem[u0 + u] = sdot * r.score.scale;
    }
  }
  __syncthreads();
}

// Warp-level bounded wait (lane 0 polls, the warp barrier orders the other
// lanes' later reads after its acquiring load).
__device__ bool warp_wait_count(const RouteParams& r, const unsigned* ctr, unsigned target) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) {
    ok = ld_relaxed(r.ctl + 2) == 0;
    if (ok && ld_acquire(ctr) < target) {
      const uint64_t t0 = global_timer_ns();
      for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if (ld_acquire(ctr) >= target) break;
        if ((it & 15u) == 0) {
          if (ld_relaxed(r.ctl + 2) != 0) { ok = 0; break; }
          if (static_cast<int64_t>(global_timer_ns() - t0) > r.limit_ns) {
            report_status(r.status, PBSA_ERR_TIMEOUT);
            atomicExch(r.ctl + 2, 1u);
            ok = 0;
            break;
          }
        }
      }
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// One function per kind of ticket.
template <int D>
__device__ __forceinline__ void ticket_plan(const RouteParams& r, int tk, uint8_t* smem) {
  // a head's update plan, with the memory scores of its items computed here
  const int bh = tk - r.t_plan;
  if (!wait_count(r, r.pool_done + bh, static_cast<unsigned>(r.per_pool))) return;
  ROUTE_TRACE(tk, 1);
  using L = PlanLayout<D>;
  plan_item_mem<D>(r, bh, smem);
  PLAN_TRACE(bh, 5);
  plan_head(r.upd, bh, *reinterpret_cast<PlanSmem*>(smem), reinterpret_cast<float*>(smem + L::kXK),
            reinterpret_cast<const float*>(smem + L::kMem));
  PLAN_TRACE(bh, 6);
  signal_done(r.plan_done + bh);
}

template <int D>
__device__ __forceinline__ void ticket_score(const RouteParams& r, int tk, uint8_t* smem) {
  // a tile of S (and the memory scores of the chunks starting in it)
  const int x = tk - r.t_score, bh = x / r.per_score, tile = x - bh * r.per_score;
  if (!wait_count(r, r.pool_done + bh, static_cast<unsigned>(r.per_pool))) return;
  ROUTE_TRACE(tk, 1);
  score_item<D, kRouteScoreTile, 2>(r.score, bh, tile % r.n_jblk, tile / r.n_jblk,
                                    reinterpret_cast<float*>(smem));
  signal_done(r.score_done + bh);
}

template <typename T>
__device__ __forceinline__ void ticket_stash(const RouteParams& r, int tk) {
  const int x = tk - r.t_stash, bh = x / r.P, s = x - bh * r.P;
  if (!wait_count(r, r.plan_done + bh, 1u)) return;
  ROUTE_TRACE(tk, 1);
  stash_item<T, 2>(r.upd, s, bh, static_cast<const T*>(r.kpool), static_cast<const T*>(r.vpool),
                static_cast<T*>(const_cast<void*>(r.stash)));
  signal_done(r.stash_done + bh);
}

template <int W, int U>
__device__ __forceinline__ void ticket_select(const RouteParams& r, int tk, uint8_t* smem) {
  // eight attended lists: scores from the tiles, the slots' lengths after the
  // update from the plan (the window's top-k is sorted before the plan is
  // done; each warp then waits for the plan only to merge in the slots)
  const int x = tk - r.t_sel, bh = x / r.per_sel, g = x - bh * r.per_sel;
  if (!wait_count(r, r.score_done + bh, static_cast<unsigned>(r.per_score))) return;
  ROUTE_TRACE(tk, 1);
  const int i = g * kRouteSelRows + (threadIdx.x >> 5);
  const bool plans = r.t_score > r.t_plan;
  auto plan_ready = [&]() { return !plans || warp_wait_count(r, r.plan_done + bh, 1u); };
  if (i < r.nQB) {
    if (r.sel.NB <= 32 * kSelBmWords)
      select_row_bitmap<W, U>(r.sel, i, bh,
                              smem + (threadIdx.x >> 5) * sel_bitmap_smem_per_warp<W>(),
                              plan_ready);
    else
      select_row<W, U>(r.sel, i, bh, plan_ready);
  }
  __syncthreads();
}

template <typename T, int D>
__device__ __forceinline__ void ticket_apply(const RouteParams& r, int tk, uint8_t* smem) {
  // one slot written as planned
  const int x = tk - r.t_apply, bh = x / r.P, s = x - bh * r.P;
  if (!wait_count(r, r.plan_done + bh, 1u)) return;
  if (!wait_count(r, r.score_done + bh, static_cast<unsigned>(r.per_score))) return;
  if (r.merge && !wait_count(r, r.stash_done + bh, static_cast<unsigned>(r.P))) return;
  ROUTE_TRACE(tk, 1);
  int* s_mref = reinterpret_cast<int*>(smem + 8 * D * sizeof(float));
  int* s_mlen = s_mref + kMaxItems;
  float* s_mw = reinterpret_cast<float*>(s_mlen + kMaxItems);
  apply_item<T, D, 4>(r.upd, s, bh, static_cast<T*>(r.kpool), static_cast<T*>(r.vpool),
                   static_cast<const T*>(r.stash), r.blk_len, r.blk_pos, r.k_bar, r.slot_src,
                   r.slot_w, reinterpret_cast<float(*)[D]>(smem), s_mref, s_mlen, s_mw);
  signal_done(r.apply_done + bh);
}

template <typename T, int D, int W, int U>
__device__ __forceinline__ void run_ticket(const RouteParams& r, int tk, uint8_t* smem) {
  if (tk < r.t_score) ticket_plan<D>(r, tk, smem);
  else if (tk < r.t_stash) ticket_score<D>(r, tk, smem);
  else if (tk < r.t_sel) ticket_stash<T>(r, tk);
  else if (tk < r.t_apply) ticket_select<W, U>(r, tk, smem);
  else ticket_apply<T, D>(r, tk, smem);
}

template <typename T, int D, int W, int U>
__global__ void __launch_bounds__(kRouteThreads, 2) route_kernel(RouteParams r) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_next[2];
  __shared__ int s_last;
  pdl_wait();
  pdl_trigger();
  const int t = threadIdx.x;
  ROUTE_TRACE_CTA(0);
  int tk = route_pool<T, D>(r, smem);
  ROUTE_TRACE_CTA(1);
  if (tk < 0) {
    if (t == 0) s_next[0] = claim(r);
    __syncthreads();
    tk = s_next[0];
    __syncthreads();
  }
  for (int it = 0; tk < r.t_end; ++it) {
    // the next ticket is claimed only when this one is done: a ticket claimed
    // early would wait behind this one while other CTAs sit idle
    run_ticket<T, D, W, U>(r, tk, smem);
    ROUTE_TRACE(tk, 2);
    if (t == 0) {
      s_next[it & 1] = claim(r);
      ROUTE_TRACE(s_next[it & 1], 0);
    }
    __syncthreads();
    tk = s_next[it & 1];
  }

  // the last CTA out leaves every counter at zero for the next call (every
  // other CTA has made its final claim and passed its last wait by then)
  __syncthreads();
  if (t == 0) {
    __threadfence();
    s_last = atomicAdd(r.ctl + 1, 1u) == gridDim.x - 1 ? 1 : 0;
  }
  __syncthreads();
  ROUTE_TRACE_CTA(2);
  if (s_last) {
    __threadfence();
    for (int w = t; w < r.n_ctl_words; w += kRouteThreads) r.ctl[w] = 0u;
    __threadfence();
  }
}

template <typename T, int D>
size_t route_smem(const RouteParams& r) {
  const int S = r.pool.stages;
  size_t m = static_cast<size_t>(S) * r.pool.bs * D * sizeof(T) + 2 * 8 * D * sizeof(float) +
             S * (sizeof(uint64_t) + sizeof(long) + 2 * sizeof(int)) + 4 * sizeof(int);
  m = std::max(m, score_smem_bytes<D, kRouteScoreTile>());
  m = std::max(m, static_cast<size_t>(kRouteSelRows) * sel_bitmap_smem_per_warp<8>());
  if (r.t_score > r.t_plan) {
    const size_t plan = PlanLayout<D>::bytes(r.P, r.upd.policy);
    m = std::max(m, plan);
    m = std::max(m, static_cast<size_t>(8) * D * sizeof(float) + 3 * kMaxItems * sizeof(int));
  }
  return m;
}

// Launch of one instantiation; returns 1 when the shape does not fit (the
// caller then runs the per-call kernels).
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
  const int G = std::max(1, std::min(std::min(per_sm, 2) * sm_count(), r.t_end));
  if (launch(kern, dim3(G), dim3(kRouteThreads), smem, s, r) != cudaSuccess) {
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

#ifdef PBSA_ROUTE_TRACE
// Copies the time stamps of the last traced call to host memory: per ticket
// (claimed, dependencies met, done, -) then per CTA (start, pooling done,
// exit, -), all in ns of the global timer.
extern "C" int pbsa_route_trace_read(void* tickets, void* ctas) {
  if (cudaMemcpyFromSymbol(tickets, pbsa::g_route_trace, sizeof(pbsa::g_route_trace)) != cudaSuccess)
    return PBSA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(ctas, pbsa::g_route_cta, sizeof(pbsa::g_route_cta)) != cudaSuccess)
    return PBSA_ERR_CUDA;
  return PBSA_OK;
}
extern "C" int pbsa_sel_trace_read(void* out) {
  if (cudaMemcpyFromSymbol(out, pbsa::g_sel_trace, sizeof(pbsa::g_sel_trace)) != cudaSuccess)
    return PBSA_ERR_CUDA;
  return PBSA_OK;
}
extern "C" int pbsa_plan_trace_read(void* out) {
  if (cudaMemcpyFromSymbol(out, pbsa::g_plan_trace, sizeof(pbsa::g_plan_trace)) != cudaSuccess)
    return PBSA_ERR_CUDA;
  return PBSA_OK;
}
#endif

extern "C" size_t pbsa_route_workspace(const pbsa_dims* d, int P, int n_cand) {
  if (d == nullptr || P < 0 || n_cand < 0 || d->B < 1 || d->H < 1) return 0;
  size_t upd = (P >= 1) ? pbsa_update_memory_workspace(d, P, n_cand) : 0;
  return pbsa::route_ctl_bytes(static_cast<long>(d->B) * d->H) + upd;
}

extern "C" int pbsa_route_step(const pbsa_dims* d, const pbsa_route_args* a, void* workspace,
                               size_t ws_bytes, void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(a != nullptr, PBSA_ERR_ARG, "route_step: args is NULL");
  PBSA_CHECK_ARG(a->Tq >= 1 && a->NB >= 1 && a->n_pool >= 0 && a->P >= 0 && a->n_cand >= 0,
                 PBSA_ERR_SHAPE, "route_step: need Tq >= 1, NB >= 1, n_pool, P, n_cand >= 0");
  PBSA_CHECK_ARG(static_cast<long>(d->B) * d->H <= 65535, PBSA_ERR_SHAPE,
                 "route_step: B*H must be <= 65535");
  const size_t need = pbsa_route_workspace(d, a->P, a->n_cand);
  PBSA_CHECK_ARG(workspace != nullptr && ws_bytes >= need && aligned(workspace, 256),
                 PBSA_ERR_WORKSPACE,
                 "route_step: workspace missing, too small or not 256-byte aligned (need " +
                     std::to_string(need) + " bytes)");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int BH = d->B * d->H;
  const size_t ctl_bytes = route_ctl_bytes(BH);
  char* ws = static_cast<char*>(workspace);
  void* upd_ws = ws + ctl_bytes;
  const size_t upd_bytes = ws_bytes - ctl_bytes;
  const bool do_update = a->P >= 1 && a->n_cand >= 1;
  const int nQB = qb_count(a->Tq, d->q_chunk, d->bs);
  const int take_max = a->k < a->n_win ? a->k : a->n_win;
  auto pick = [](int n) { return n <= 64 ? 2 : (n <= 128 ? 4 : (n <= 256 ? 8 : 16)); };
  const int W = pick(a->n_win), U = pick(a->n_mem + take_max);

  // the per-call path: the three entry points in order (they validate their
  // own arguments); used when the fused kernel has no instantiation for this
  // shape
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
    PBSA_CHECK_ARG(d->q_chunk == 0 || d->q_chunk >= a->Tq, PBSA_ERR_SHAPE,
                   "route_step: a memory update needs a single query chunk (q_chunk 0 or >= Tq)");
  }
  const int n_jblk = (a->NB + kRouteScoreTile - 1) / kRouteScoreTile;
  const int n_itile = (nQB + kRouteScoreTile - 1) / kRouteScoreTile;
  const int per_sel = (nQB + kRouteSelRows - 1) / kRouteSelRows;
  const int P_upd = do_update ? a->P : 0;
  const bool merge = do_update && a->policy == PBSA_MERGE_MEAN;
  const long per_pool = static_cast<long>(nQB) + a->n_pool;
  const long n_tickets = static_cast<long>(BH) *
                         (per_pool + static_cast<long>(n_jblk) * n_itile + (do_update ? 1 : 0) +
                          (merge ? P_upd : 0) + P_upd + per_sel);
  PBSA_CHECK_ARG(n_tickets < (1L << 30), PBSA_ERR_SHAPE, "route_step: too much work for one call");
  int* status = device_status_ptr();
  PBSA_CHECK_ARG(status != nullptr, PBSA_ERR_CUDA, "route_step: no device status word");

  RouteParams r;
  r.pool.q = a->q; r.pool.kpool = a->kpool; r.pool.blk_len = a->blk_len;
  r.pool.pool_ids = a->pool_ids; r.pool.q_bar = a->q_bar; r.pool.k_bar = a->k_bar;
  r.pool.Tq = a->Tq; r.pool.qc = d->q_chunk; r.pool.NB = a->NB; r.pool.bs = d->bs;
  r.pool.nQB = nQB; r.pool.n_pool = a->n_pool;
  r.pool.n_items = static_cast<int>(BH * per_pool);
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
  if (do_update) {
    // the plan's statement of each slot's length and position after the update
    const dev::PlanView pv0 = dev::plan_view(upd_ws, 0, a->P, a->P + a->n_cand);
    r.sel.slot_len = pv0.nlen;
    r.sel.slot_pos = pv0.npos;
    r.sel.slot_ld = static_cast<long>(dev::plan_bytes(a->P, a->P + a->n_cand) / 4);
    r.sel.n_slot = a->P;
  } else {
    r.sel.slot_len = nullptr; r.sel.slot_pos = nullptr; r.sel.slot_ld = 0; r.sel.n_slot = 0;
  }
  r.kpool = a->kpool; r.vpool = a->vpool;
  r.stash = do_update ? static_cast<const char*>(upd_ws) +
                            static_cast<size_t>(BH) * dev::plan_bytes(a->P, a->P + a->n_cand)
                      : nullptr;
  r.blk_len = a->blk_len; r.blk_pos = a->blk_pos; r.k_bar = a->k_bar;
  r.slot_src = a->slot_src; r.slot_w = a->slot_w;
  r.ctl = reinterpret_cast<unsigned*>(ws);
  r.pool_done = r.ctl + kCtlWords;
  r.score_done = r.pool_done + BH;
  r.plan_done = r.score_done + BH;
  r.stash_done = r.plan_done + BH;
  r.apply_done = r.stash_done + BH;
  r.n_ctl_words = kCtlWords + 5 * BH;
  r.BH = BH; r.P = a->P; r.nQB = nQB; r.n_jblk = n_jblk; r.n_itile = n_itile;
  r.per_pool = static_cast<int>(per_pool);
  r.per_score = n_jblk * n_itile;
  r.per_sel = per_sel;
  r.merge = merge ? 1 : 0;
  // ticket order: pool, plan, score, stash, select, apply (every ticket's
  // dependencies come before it)
  r.t_plan = static_cast<int>(BH * per_pool);
  r.t_score = r.t_plan + (do_update ? BH : 0);
  r.t_stash = r.t_score + BH * r.per_score;
  r.t_sel = r.t_stash + (merge ? BH * P_upd : 0);
  r.t_apply = r.t_sel + BH * per_sel;
  r.t_end = r.t_apply + BH * P_upd;
  r.status = status; r.limit_ns = wait_limit_ns(); r.debug = debug_flags();

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
