// Device code of a3, the persistent-memory update, shared by the per-call
// kernels (update.cu) and the fused routing kernel (route.cu).
//
// Top-C retention with sinks; evict or mean-merge the losers, written into the
// slot ids 0..P-1 of the block pool in place.  Sparse Forcing keeps a bounded
// memory of historical blocks: sink anchors plus dynamic blocks chosen by
// coarse scoring, refreshed with Top-C retention as blocks leave the local
// window (gist.science/es, section 2 "Arquitectura Propuesta"); the abstract
// adds that the memory compresses persistent blocks as well as keeping them;
// PBSA item "Optimización" names selective cache updates as part of the
// kernel's job.
//
//   plan_head   one (b,h): rank the candidates by their unique 64-bit keys
//               (each thread counts the larger keys), assign slots, choose
//               merge targets by pooled-key dot products, and write a per-slot
//               plan into the workspace;
//   stash_item  (merge policy only) copy the old content of a losing slot that
//               is about to be overwritten and is still needed by a merge;
//   apply_item  one (slot, b, h): write the slot's new rows (copy or weighted
//               mean), recompute its pooled key, update its metadata.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"

// Optional time stamps inside plan_head for schedule studies (the fused
// routing kernel defines this when built with -DPBSA_ROUTE_TRACE).
#ifndef PLAN_TRACE
#define PLAN_TRACE(bh, k) do {} while (0)
#endif

namespace pbsa {
namespace dev {

constexpr int kMaxItems = 256;
constexpr int OP_NONE = 0, OP_WRITE = 1, OP_CLEAR = 2;

struct PlanView {
  int32_t* op;        // [P]
  int32_t* base;      // [P] physical id of the base content
  int32_t* base_len;  // [P]
  int32_t* src;       // [P] global id of the slot's block
  int32_t* pos;       // [P]
  int32_t* stash;     // [P] 1: copy slot s to the stash before it is overwritten
  int32_t* moff;      // [P + 1] merge list offsets
  int32_t* mref;      // [M] physical id, or -(1 + s) for stash entry s
  int32_t* mlen;      // [M]
  int32_t* nlen;      // [P] the slot's blk_len after the update
  int32_t* npos;      // [P] the slot's blk_pos after the update
  float* base_w;      // [P]
  float* mw;          // [M]
};

__host__ __device__ inline size_t plan_bytes(int P, int M) {
  size_t ints = 9 * static_cast<size_t>(P) + 1 + 2 * static_cast<size_t>(M);
  size_t flts = static_cast<size_t>(P) + static_cast<size_t>(M);
  return ((ints + flts) * 4 + 255) / 256 * 256;
}

__host__ __device__ inline PlanView plan_view(void* ws, long bh, int P, int M) {
  char* p = static_cast<char*>(ws) + bh * plan_bytes(P, M);
  int32_t* ip = reinterpret_cast<int32_t*>(p);
  PlanView v;
  v.op = ip; ip += P;
  v.base = ip; ip += P;
  v.base_len = ip; ip += P;
  v.src = ip; ip += P;
  v.pos = ip; ip += P;
  v.stash = ip; ip += P;
  v.moff = ip; ip += P + 1;
  v.mref = ip; ip += M;
  v.mlen = ip; ip += M;
  v.nlen = ip; ip += P;
  v.npos = ip; ip += P;
  float* fp = reinterpret_cast<float*>(ip);
  v.base_w = fp; fp += P;
  v.mw = fp;
  return v;
}

struct UpdArgs {
  int B, H, D, bs, NB, P, n_sink, n_cand, policy, M;
  const int32_t* blk_len;
  const int32_t* blk_pos;
  const float* k_bar;
  const int32_t* slot_src;
  const float* slot_w;
  const int32_t* cand_ids;
  const int32_t* cand_src;
  const float* mem;
  void* ws;
  int* status;
};

// Exclusive prefix sum of one value per thread over a 256-thread CTA (all
// threads call it; it synchronises the CTA).  `total` (if given) receives the
// sum over all threads.
__device__ __forceinline__ int block_excl_scan256(int v, int* tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += u;
  }
  if (lane == 31) tot[warp] = incl;
  __syncthreads();
  int base = 0, all = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const int x = tot[w];
    base += w < warp ? x : 0;
    all += x;
  }
  __syncthreads();
  if (total) *total = all;
  return base + incl - v;
}

// --------------------------------------------------------------------- plan
// Dynamic shared memory of plan_head under the merge policy: the kept slots'
// pooled keys (padded rows) and one loser key per warp.
__host__ __device__ inline size_t merge_key_smem(int P, int D) {
  return (static_cast<size_t>(P) * (D / 4 + 1) + 8 * static_cast<size_t>(D / 4)) * 16;
}

// Shared memory of plan_head (one (b,h) at a time, 256 threads).
struct __align__(16) PlanSmem {
  uint64_t skey[kMaxItems];
  int it_phys[kMaxItems], it_src[kMaxItems], it_old[kMaxItems], it_len[kMaxItems];
  int it_pos[kMaxItems];
  float it_w[kMaxItems];
  int it_slot[kMaxItems];      // slot it occupies after the update (kept) or -1
  int it_target[kMaxItems];    // merge target slot (losers) or -1
  int it_rank[kMaxItems];      // position in the ranking
  int holder[256];             // item held by slot s after the update
  int free_pos[256];
  int sink_item[256];
  int tcount[256];
  int tmaxlen[256];            // longest loser merged into slot s
  int s_op[256];
  int s_moff[256];
  int s_tot[8];
  int s_nvalid;
};

// The update plan of head bh, written to its part of the workspace.  `sk`
// holds P*D floats (kept pooled keys, merge policy only).  `item_mem`, if not
// NULL, holds the memory score of every plan item (occupied non-sink slots,
// then the candidates), computed by the caller; otherwise they are read from
// a.mem.
__device__ inline void plan_head(const UpdArgs& a, long bh, PlanSmem& sm, float* sk,
                                 const float* item_mem = nullptr) {
  uint64_t* skey = sm.skey;
  int* it_phys = sm.it_phys;
  int* it_src = sm.it_src;
  int* it_old = sm.it_old;
  int* it_len = sm.it_len;
  int* it_pos = sm.it_pos;
  float* it_w = sm.it_w;
  int* it_slot = sm.it_slot;
  int* it_target = sm.it_target;
  int* it_rank = sm.it_rank;
  int* holder = sm.holder;
  int* free_pos = sm.free_pos;
  int* sink_item = sm.sink_item;
  int* tcount = sm.tcount;
  int* tmaxlen = sm.tmaxlen;
  int* s_op = sm.s_op;
  int* s_moff = sm.s_moff;
  int* s_tot = sm.s_tot;
  int& s_nvalid = sm.s_nvalid;
  __syncthreads();   // shared memory may still be read by the previous item
  PLAN_TRACE(bh, 0);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int P = a.P, n_sink = a.n_sink;
  const int n_dyn = P - n_sink;
  const int NI = n_dyn + a.n_cand;
  PlanView pv = plan_view(a.ws, bh, P, a.M);

  // ---- candidates
  for (int s = t; s < P; s += 256) { holder[s] = -1; sink_item[s] = -1; }
  __syncthreads();
  if (t < kMaxItems) {
    it_slot[t] = -1;
    it_target[t] = -1;
    it_rank[t] = -1;
    uint64_t key = 0;
    int phys = -1, src = -1, old = -1, len = 0;
    float w = 0.f;
    bool valid = false;
    if (t < n_dyn) {
      const int s = n_sink + t;
      src = a.slot_src[bh * P + s];
      if (src >= 0) {
        valid = true;
        phys = s; old = s; w = a.slot_w[bh * P + s];
      }
    } else if (t < NI) {
      const int c = t - n_dyn;
      phys = a.cand_ids[c];
      src = a.cand_src[c];
      if (phys < 0 || phys >= a.NB || src < 0 || src >= (1 << 24)) {
        report_status(a.status, PBSA_ERR_ARG);
        phys = -1;
      } else if (src < n_sink) {
        sink_item[src] = t;       // fills its sink slot, not ranked
      } else {
        valid = true; w = 1.f;
      }
    }
    int pos = 0;
    if (phys >= 0) {
      len = a.blk_len[bh * a.NB + phys];
      pos = a.blk_pos[bh * a.NB + phys];
    }
    it_pos[t] = pos;
    if (valid) {
      const float m = item_mem ? item_mem[t] : a.mem[bh * a.NB + phys];
      key = (static_cast<uint64_t>(orderable(m)) << 32) |
            (static_cast<uint64_t>(0xffffffu - static_cast<uint32_t>(src)) << 8) |
            static_cast<uint64_t>(t);
    }
    it_phys[t] = phys; it_src[t] = src; it_old[t] = old; it_len[t] = len; it_w[t] = w;
    skey[t] = key;
  }
  __syncthreads();

  // ---- rank: keys are unique (item index in the low bits), so an item's
  PLAN_TRACE(bh, 1);
  // position in the descending order is the number of larger keys; all 256
  // threads count at once.
  {
    const uint64_t mine = skey[t];
    int rank = 0;
    // keys past NI are zero and never larger; 8 keys per step, all loads first
    const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(skey);
    for (int u2 = 0; u2 < (NI + 7) / 8 * 4; u2 += 4) {
      ulonglong2 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = k2[u2 + q];
#pragma unroll
      for (int q = 0; q < 4; ++q) rank += (v[q].x > mine ? 1 : 0) + (v[q].y > mine ? 1 : 0);
    }
    if (mine != 0) it_rank[t] = rank;
    const int nv = __syncthreads_count(mine != 0 ? 1 : 0);
    if (t == 0) s_nvalid = nv;
  }
  __syncthreads();
  const int n_valid = s_nvalid;
  const int n_keep = min(n_dyn, n_valid);

  // ---- kept old slots stay; list the free non-sink slots in ascending order
  PLAN_TRACE(bh, 2);
  if (t < NI && it_rank[t] >= 0 && it_rank[t] < n_keep && it_old[t] >= 0) {
    it_slot[t] = it_old[t];
    holder[it_old[t]] = t;
  }
  __syncthreads();
  {
    const int f = (t >= n_sink && t < P && holder[t] < 0) ? 1 : 0;
    const int at = block_excl_scan256(f, s_tot, nullptr);
    if (f) free_pos[at] = t;
  }
  __syncthreads();
  // newly kept blocks take free slots in ascending global-id order.  When the
  // candidates' global ids ascend with their list position (the usual case:
  // a chunk's blocks in order), that order is the item order and a prefix
  // count gives each block its free slot; otherwise every block counts the
  // kept new blocks with smaller ids.
  {
    const bool is_new_kept = t < NI && it_rank[t] >= 0 && it_rank[t] < n_keep && it_old[t] < 0;
    const bool ascending =
        __syncthreads_and(!(t > n_dyn && t < NI && it_src[t - 1] >= it_src[t])) != 0;
    if (ascending) {
      const int r = block_excl_scan256(is_new_kept ? 1 : 0, s_tot, nullptr);
      if (is_new_kept) {
        it_slot[t] = free_pos[r];
        holder[free_pos[r]] = t;
      }
    } else if (is_new_kept) {
      int r = 0;
      for (int u = 0; u < NI; ++u)
        if (it_rank[u] >= 0 && it_rank[u] < n_keep && it_old[u] < 0 && it_src[u] < it_src[t]) ++r;
      it_slot[t] = free_pos[r];
      holder[free_pos[r]] = t;
    }
  }
  __syncthreads();

  // ---- merge targets: most similar kept slot by pooled-key dot product
  PLAN_TRACE(bh, 3);
  // (ties -> lowest slot).  The kept blocks' pooled keys are staged in shared
  // memory with a padded row stride; each warp takes one loser at a time, its
  // lanes take one slot each (a full dot product over D, in dimension order),
  // and a warp argmax picks the target.
  if (a.policy == PBSA_MERGE_MEAN && n_keep > 0) {
    const int D4 = a.D / 4;
    const int ST4 = D4 + 1;                          // padded row stride (float4)
    float4* sk4 = reinterpret_cast<float4*>(sk);     // [P][ST4]
    float4* kw = sk4 + P * ST4 + warp * D4;          // this warp's loser key
    const float4* kb4 = reinterpret_cast<const float4*>(a.k_bar);
    for (int e0 = 0; e0 < P * D4; e0 += 256 * 4) {
      float4 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = e0 + q * 256 + t;
        const int s = e / D4;
        const int c = (e < P * D4 && s >= n_sink) ? holder[s] : -1;
        v[q] = c >= 0 ? kb4[(bh * a.NB + it_phys[c]) * D4 + e % D4] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = e0 + q * 256 + t;
        if (e < P * D4) sk4[(e / D4) * ST4 + e % D4] = v[q];
      }
    }
    __syncthreads();
    for (int u = warp; u < NI; u += 8) {
      if (!(it_rank[u] >= n_keep)) continue;          // losers only (warp-uniform)
      if (lane < D4) kw[lane] = kb4[(bh * a.NB + it_phys[u]) * D4 + lane];
      __syncwarp();
      float best = -INFINITY;
      int best_s = -1;
      for (int s0 = n_sink; s0 < P; s0 += 32) {
        const int s = s0 + lane;
        const bool valid = s < P && holder[s] >= 0;
        float dot = 0.f;
        if (s < P) {
          const float4* kc = sk4 + s * ST4;
          for (int d4 = 0; d4 < D4; ++d4) {
            const float4 x = kw[d4], y = kc[d4];
            dot = fmaf(x.x, y.x, dot);
            dot = fmaf(x.y, y.y, dot);
            dot = fmaf(x.z, y.z, dot);
            dot = fmaf(x.w, y.w, dot);
          }
        }
        float v = valid ? dot : -INFINITY;
        int si = valid ? s : 0x7fffffff;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, v, off);
          const int os = __shfl_xor_sync(0xffffffffu, si, off);
          if (ov > v || (ov == v && os < si)) {
            v = ov;
            si = os;
          }
        }
        if (si != 0x7fffffff && (v > best || best_s < 0)) {
          best = v;
          best_s = si;
        }
      }
      if (lane == 0) it_target[u] = best_s;
      __syncwarp();
    }
  }
  // merge lists grouped by target slot, each in ranking order (deterministic
  // summation order): the losers are listed by rank, then one warp per target
  // slot counts (and later places) its losers with ballots
  const bool merging = a.policy == PBSA_MERGE_MEAN && n_keep > 0;
  const int n_lose = n_valid - n_keep;
  int* rank_item = free_pos;                 // free_pos is no longer needed
  if (merging && t < NI && it_rank[t] >= n_keep) rank_item[it_rank[t] - n_keep] = t;
  __syncthreads();
  for (int s = warp; s < P; s += 8) {
    int n = 0, mx = 0;
    if (merging) {
      for (int c0 = 0; c0 < n_lose; c0 += 32) {
        const int u = c0 + lane < n_lose ? rank_item[c0 + lane] : -1;
        const bool hit = u >= 0 && it_target[u] == s;
        n += __popc(__ballot_sync(0xffffffffu, hit));
        mx = max(mx, __reduce_max_sync(0xffffffffu, hit ? it_len[u] : 0));
      }
    }
    if (lane == 0) {
      tcount[s] = n;
      tmaxlen[s] = mx;
    }
  }
  __syncthreads();

  // ---- per-slot plan (thread s plans slot s)
  PLAN_TRACE(bh, 4);
  if (t < P) {
    const int s = t;
    int op = OP_NONE, base = -1, blen = 0, src = -1, pos = 0;
    float bw = 0.f;
    if (s < n_sink) {
      const int u = sink_item[s];
      if (u >= 0) {
        op = OP_WRITE; base = it_phys[u]; blen = it_len[u]; bw = 1.f; src = s;
        pos = it_pos[u];
      }
    } else {
      const int c = holder[s];
      if (c < 0) {
        op = OP_CLEAR;
      } else {
        base = it_phys[c]; blen = it_len[c]; bw = it_w[c]; src = it_src[c];
        pos = it_pos[c];
        op = (it_old[c] < 0 || tcount[s] > 0) ? OP_WRITE : OP_NONE;
      }
    }
    s_op[s] = op;
    pv.op[s] = op; pv.base[s] = base; pv.base_len[s] = blen; pv.base_w[s] = bw;
    pv.src[s] = src; pv.pos[s] = pos; pv.stash[s] = 0;
    // what apply_item will leave in blk_len / blk_pos of the slot
    int nl = 0, np = 0;
    if (op == OP_NONE) {
      nl = a.blk_len[bh * a.NB + s];
      np = a.blk_pos[bh * a.NB + s];
    } else if (op == OP_WRITE) {
      nl = tcount[s] > 0 ? max(blen, tmaxlen[s]) : blen;
      np = pos;
    }
    pv.nlen[s] = nl;
    pv.npos[s] = np;
  }
  const int v = (t < P) ? tcount[t] : 0;
  int total = 0;
  const int moff = block_excl_scan256(v, s_tot, &total);   // synchronises: s_op complete
  if (t < P) {
    pv.moff[t] = moff;
    s_moff[t] = moff;
  }
  if (t == 0) pv.moff[P] = total;
  // losers that are old slots overwritten by a new block are read from the stash
  if (t < NI && it_target[t] >= 0 && it_old[t] >= 0 && s_op[it_old[t]] == OP_WRITE)
    pv.stash[it_old[t]] = 1;
  __syncthreads();
  if (merging) {
    for (int s = warp; s < P; s += 8) {
      int base = s_moff[s];
      for (int c0 = 0; c0 < n_lose; c0 += 32) {
        const int u = c0 + lane < n_lose ? rank_item[c0 + lane] : -1;
        const bool hit = u >= 0 && it_target[u] == s;
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (hit) {
          const int slot = base + __popc(m & ((1u << lane) - 1u));
          const int old = it_old[u];
          const bool from_stash = old >= 0 && s_op[old] == OP_WRITE;
          pv.mref[slot] = from_stash ? -(1 + old) : it_phys[u];
          pv.mlen[slot] = it_len[u];
          pv.mw[slot] = it_w[u];
        }
        base += __popc(m);
      }
    }
  }
}

// -------------------------------------------------------------------- stash
// Copy slot s of head bh to the stash when the plan asks for it.
// CB: 16-byte chunks of K and of V each thread holds per round (the fused
// routing kernel runs with fewer registers and passes a smaller batch).
template <typename T, int CB = 8>
__device__ void stash_item(const UpdArgs& a, int s, long bh, const T* __restrict__ kpool,
                           const T* __restrict__ vpool, T* __restrict__ stash) {
  PlanView pv = plan_view(a.ws, bh, a.P, a.M);
  if (!pv.stash[s]) return;
  const int n16 = static_cast<int>(static_cast<long>(a.bs) * a.D * sizeof(T) / 16);
  const uint4* ks = reinterpret_cast<const uint4*>(kpool + (bh * a.NB + s) * static_cast<long>(a.bs) * a.D);
  const uint4* vs = reinterpret_cast<const uint4*>(vpool + (bh * a.NB + s) * static_cast<long>(a.bs) * a.D);
  uint4* kd = reinterpret_cast<uint4*>(stash + ((bh * a.P + s) * 2 + 0) * static_cast<long>(a.bs) * a.D);
  uint4* vd = reinterpret_cast<uint4*>(stash + ((bh * a.P + s) * 2 + 1) * static_cast<long>(a.bs) * a.D);
  for (int e0 = 0; e0 < n16; e0 += 256 * CB) {
    uint4 ka[CB], va[CB];
#pragma unroll
    for (int k = 0; k < CB; ++k) {
      const int e = e0 + threadIdx.x + k * 256;
      if (e < n16) { ka[k] = ks[e]; va[k] = vs[e]; }
    }
#pragma unroll
    for (int k = 0; k < CB; ++k) {
      const int e = e0 + threadIdx.x + k * 256;
      if (e < n16) { kd[e] = ka[k]; vd[e] = va[k]; }
    }
  }
}

// -------------------------------------------------------------------- apply
template <typename T>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int EPC = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&x)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
    x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z); x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
  }
  __device__ static uint4 raw(const __nv_bfloat16* p) { return *reinterpret_cast<const uint4*>(p); }
  __device__ static void fma_raw(float w, uint4 u, float (&acc)[8]) {
    acc[0] = fmaf(w, bf16_lo(u.x), acc[0]); acc[1] = fmaf(w, bf16_hi(u.x), acc[1]);
    acc[2] = fmaf(w, bf16_lo(u.y), acc[2]); acc[3] = fmaf(w, bf16_hi(u.y), acc[3]);
    acc[4] = fmaf(w, bf16_lo(u.z), acc[4]); acc[5] = fmaf(w, bf16_hi(u.z), acc[5]);
    acc[6] = fmaf(w, bf16_lo(u.w), acc[6]); acc[7] = fmaf(w, bf16_hi(u.w), acc[7]);
  }
  // rounds to storage, stores, and returns the stored values in x
  __device__ static void store(__nv_bfloat16* p, float (&x)[8]) {
    uint4 u;
    u.x = pack_bf16x2(x[0], x[1]); u.y = pack_bf16x2(x[2], x[3]);
    u.z = pack_bf16x2(x[4], x[5]); u.w = pack_bf16x2(x[6], x[7]);
    *reinterpret_cast<uint4*>(p) = u;
    x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
    x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z); x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
  }
};
template <>
struct Elem<float> {
  static constexpr int EPC = 4;
  __device__ static void load(const float* p, float (&x)[4]) {
    float4 u = *reinterpret_cast<const float4*>(p);
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
  }
  __device__ static uint4 raw(const float* p) { return *reinterpret_cast<const uint4*>(p); }
  __device__ static void fma_raw(float w, uint4 u, float (&acc)[4]) {
    acc[0] = fmaf(w, __uint_as_float(u.x), acc[0]); acc[1] = fmaf(w, __uint_as_float(u.y), acc[1]);
    acc[2] = fmaf(w, __uint_as_float(u.z), acc[2]); acc[3] = fmaf(w, __uint_as_float(u.w), acc[3]);
  }
  __device__ static void store(float* p, float (&x)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
};

// Write slot s of head bh as planned (copy, weighted mean or clear) and update
// its pooled key and metadata.  A plain copy moves CB 16-byte chunks of K and
// of V per thread per round.  `red` holds 8*D floats; s_mref, s_mlen and
// s_mw are shared arrays of kMaxItems entries for the slot's merge list.
template <typename T, int D, int CB = 8>
__device__ void apply_item(const UpdArgs& a, int s, long bh, T* __restrict__ kpool,
                           T* __restrict__ vpool, const T* stash,
                           int32_t* __restrict__ blk_len, int32_t* __restrict__ blk_pos,
                           float* __restrict__ k_bar, int32_t* __restrict__ slot_src,
                           float* __restrict__ slot_w, float (*red)[D], int* s_mref,
                           int* s_mlen, float* s_mw) {
  constexpr int EPC = Elem<T>::EPC;
  constexpr int CPR = D / EPC;
  constexpr int RPP = 256 / CPR;
  __syncthreads();   // `red` may still be read by the previous item
  const int t = threadIdx.x;
  PlanView pv = plan_view(a.ws, bh, a.P, a.M);
  // every plan field of this slot in one round of loads
  const int op = pv.op[s];
  const int base = pv.base[s];
  const int m0 = pv.moff[s], m1 = pv.moff[s + 1];
  const int blen = pv.base_len[s];
  const float bw = pv.base_w[s];
  const int psrc = pv.src[s], ppos = pv.pos[s];
  if (op == OP_NONE) return;
  const long blk_elems = static_cast<long>(a.bs) * D;
  float* kb_out = k_bar + (bh * a.NB + s) * static_cast<long>(D);
  if (op == OP_CLEAR) {
    if (t == 0) {
      slot_src[bh * a.P + s] = -1;
      slot_w[bh * a.P + s] = 0.f;
      blk_len[bh * a.NB + s] = 0;
      blk_pos[bh * a.NB + s] = 0;
    }
    if (t < D) kb_out[t] = 0.f;
    return;
  }
  T* kd = kpool + (bh * a.NB + s) * blk_elems;
  T* vd = vpool + (bh * a.NB + s) * blk_elems;
  const T* kb = kpool + (bh * a.NB + base) * blk_elems;
  const T* vb = vpool + (bh * a.NB + base) * blk_elems;
  if (m0 == m1) {
    // plain copy of a newly admitted block (base != s)
    // source and destination are different blocks of the same pool: load a
    // batch of 16-byte chunks into registers, then store them
    const int n16 = static_cast<int>(blk_elems * sizeof(T) / 16);
    for (int e0 = 0; e0 < n16; e0 += 256 * CB) {
      uint4 ka[CB], va[CB];
#pragma unroll
      for (int k = 0; k < CB; ++k) {
        const int e = e0 + t + k * 256;
        if (e < n16) {
          ka[k] = reinterpret_cast<const uint4*>(kb)[e];
          va[k] = reinterpret_cast<const uint4*>(vb)[e];
        }
      }
#pragma unroll
      for (int k = 0; k < CB; ++k) {
        const int e = e0 + t + k * 256;
        if (e < n16) {
          reinterpret_cast<uint4*>(kd)[e] = ka[k];
          reinterpret_cast<uint4*>(vd)[e] = va[k];
        }
      }
    }
    if (t < D) kb_out[t] = a.k_bar[(bh * a.NB + base) * static_cast<long>(D) + t];
    if (t == 0) {
      slot_src[bh * a.P + s] = psrc;
      slot_w[bh * a.P + s] = bw;
      blk_len[bh * a.NB + s] = blen;
      blk_pos[bh * a.NB + s] = ppos;
    }
    return;
  }
  // weighted row-wise mean of the base and its merged losers.  The merge list
  // is read into shared memory once; rows are processed RG row passes at a
  // time so that all loads of one merge source are in flight together.
  const int nm = m1 - m0;
  for (int m = t; m < nm; m += 256) {
    s_mref[m] = pv.mref[m0 + m];
    s_mlen[m] = pv.mlen[m0 + m];
    s_mw[m] = pv.mw[m0 + m];
  }
  __syncthreads();
  float wsum = bw;
  int nlen = blen;
  for (int m = 0; m < nm; ++m) {
    wsum += s_mw[m];
    nlen = max(nlen, s_mlen[m]);
  }
  const float inv = 1.f / wsum;
  const int c = t % CPR, rg = t / CPR;
  constexpr int RG = 2;
  float colsum[EPC];
#pragma unroll
  for (int e = 0; e < EPC; ++e) colsum[e] = 0.f;
  for (int r0 = rg; r0 < a.bs; r0 += RG * RPP) {
    float ak[RG][EPC], av[RG][EPC];
#pragma unroll
    for (int i = 0; i < RG; ++i) {
      const int r = r0 + i * RPP;
      const long off = static_cast<long>(r) * D + c * EPC;
      float xk[EPC], xv[EPC];
#pragma unroll
      for (int e = 0; e < EPC; ++e) { xk[e] = 0.f; xv[e] = 0.f; }
      if (r < a.bs && r < blen) {
        Elem<T>::load(kb + off, xk);
        Elem<T>::load(vb + off, xv);
      }
#pragma unroll
      for (int e = 0; e < EPC; ++e) {
        ak[i][e] = r < blen ? bw * xk[e] : 0.f;
        av[i][e] = r < blen ? bw * xv[e] : 0.f;
      }
    }
    for (int m = 0; m < nm; ++m) {
      const int ref = s_mref[m];
      const int ml = s_mlen[m];
      const float w = s_mw[m];
      const T* ks;
      const T* vs;
      if (ref >= 0) {
        ks = kpool + (bh * a.NB + ref) * blk_elems;
        vs = vpool + (bh * a.NB + ref) * blk_elems;
      } else {
        const int so = -(ref + 1);
        ks = stash + ((bh * a.P + so) * 2 + 0) * blk_elems;
        vs = stash + ((bh * a.P + so) * 2 + 1) * blk_elems;
      }
      uint4 xk[RG], xv[RG];
#pragma unroll
      for (int i = 0; i < RG; ++i) {
        const int r = r0 + i * RPP;
        if (r < a.bs && r < ml) {
          const long off = static_cast<long>(r) * D + c * EPC;
          xk[i] = Elem<T>::raw(ks + off);
          xv[i] = Elem<T>::raw(vs + off);
        }
      }
#pragma unroll
      for (int i = 0; i < RG; ++i) {
        const int r = r0 + i * RPP;
        if (r < a.bs && r < ml) {
          Elem<T>::fma_raw(w, xk[i], ak[i]);
          Elem<T>::fma_raw(w, xv[i], av[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < RG; ++i) {
      const int r = r0 + i * RPP;
      if (r >= a.bs) continue;
      const long off = static_cast<long>(r) * D + c * EPC;
#pragma unroll
      for (int e = 0; e < EPC; ++e) { ak[i][e] *= inv; av[i][e] *= inv; }
      // every thread reads its own elements above before writing them here
      Elem<T>::store(kd + off, ak[i]);
      Elem<T>::store(vd + off, av[i]);
      if (r < nlen) {
#pragma unroll
        for (int e = 0; e < EPC; ++e) colsum[e] += ak[i][e];
      }
    }
  }
#pragma unroll
  for (int off = CPR; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < EPC; ++e) colsum[e] += __shfl_xor_sync(0xffffffffu, colsum[e], off);
  }
  const int lane = t & 31, warp = t >> 5;
  if (lane < CPR) {
#pragma unroll
    for (int e = 0; e < EPC; ++e) red[warp][lane * EPC + e] = colsum[e];
  }
  __syncthreads();
  if (t < D) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) sum += red[w][t];
    kb_out[t] = sum / static_cast<float>(nlen);
  }
  if (t == 0) {
    slot_src[bh * a.P + s] = psrc;
    slot_w[bh * a.P + s] = wsum;
    blk_len[bh * a.NB + s] = nlen;
    blk_pos[bh * a.NB + s] = ppos;
  }
}


inline size_t stash_bytes(const pbsa_dims* d, int P) {
  return align_up(static_cast<size_t>(d->B) * d->H * P * 2 * d->bs * d->D * elem_size(d->dtype),
                  256);
}

}  // namespace dev
}  // namespace pbsa
