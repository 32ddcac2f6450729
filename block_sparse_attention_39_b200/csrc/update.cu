// a3: persistent-memory update (Top-C retention with sinks; evict or
// mean-merge the losers), written into the slot ids 0..P-1 of the block pool
// in place.
//
// Sparse Forcing keeps a bounded memory P_t of historical blocks: sink anchors
// plus dynamic blocks chosen by coarse scoring, refreshed with Top-C retention
// as blocks leave the local window (gist.science/es, section 2 "Arquitectura
// Propuesta"); the abstract adds that the memory compresses persistent blocks
// as well as keeping them; PBSA item "Optimización" names selective cache
// updates as part of the kernel's job.
//
// Three launches:
//   plan   one CTA per (b,h): rank the candidates by their unique 64-bit keys
//          (each thread counts the larger keys), assign slots, choose merge targets by pooled-key dot
//          products, and write a per-slot plan into the workspace;
//   stash  (merge policy only) copy the old content of every losing slot that
//          is about to be overwritten and is still needed by a merge;
//   apply  one CTA per (slot, b, h): write the slot's new rows (copy or
//          weighted mean), recompute its pooled key, update its metadata.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace pbsa {
namespace {

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
  float* base_w;      // [P]
  float* mw;          // [M]
};

__host__ __device__ inline size_t plan_bytes(int P, int M) {
  size_t ints = 7 * static_cast<size_t>(P) + 1 + 2 * static_cast<size_t>(M);
  size_t flts = static_cast<size_t>(P) + static_cast<size_t>(M);
  return ((ints + flts) * 4 + 255) / 256 * 256;
}

__device__ inline PlanView plan_view(void* ws, long bh, int P, int M) {
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

// --------------------------------------------------------------------- plan
__global__ void __launch_bounds__(256) update_plan_kernel(UpdArgs a) {
  __shared__ uint64_t skey[kMaxItems];
  __shared__ int it_phys[kMaxItems], it_src[kMaxItems], it_old[kMaxItems], it_len[kMaxItems];
  __shared__ float it_w[kMaxItems];
  __shared__ int it_slot[kMaxItems];      // slot it occupies after the update (kept) or -1
  __shared__ int it_target[kMaxItems];    // merge target slot (losers) or -1
  __shared__ int it_rank[kMaxItems];      // position in the ranking
  __shared__ int holder[256];             // item held by slot s after the update
  __shared__ int free_pos[256];
  __shared__ int sink_item[256];
  __shared__ int s_nvalid;

  const long bh = blockIdx.x;
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
    if (phys >= 0) len = a.blk_len[bh * a.NB + phys];
    if (valid) {
      const float m = a.mem[bh * a.NB + phys];
      key = (static_cast<uint64_t>(orderable(m)) << 32) |
            (static_cast<uint64_t>(0xffffffu - static_cast<uint32_t>(src)) << 8) |
            static_cast<uint64_t>(t);
    }
    it_phys[t] = phys; it_src[t] = src; it_old[t] = old; it_len[t] = len; it_w[t] = w;
    skey[t] = key;
  }
  __syncthreads();

  // ---- rank: keys are unique (item index in the low bits), so an item's
  // position in the descending order is the number of larger keys; all 256
  // threads count at once.
  {
    const uint64_t mine = skey[t];
    int rank = 0;
    for (int u = 0; u < NI; ++u) rank += skey[u] > mine ? 1 : 0;
    if (mine != 0) it_rank[t] = rank;
    const int nv = __syncthreads_count(mine != 0 ? 1 : 0);
    if (t == 0) s_nvalid = nv;
  }
  __syncthreads();
  const int n_valid = s_nvalid;
  const int n_keep = min(n_dyn, n_valid);

  // ---- kept old slots stay; list the free non-sink slots in ascending order
  if (t < NI && it_rank[t] >= 0 && it_rank[t] < n_keep && it_old[t] >= 0) {
    it_slot[t] = it_old[t];
    holder[it_old[t]] = t;
  }
  __syncthreads();
  if (t == 0) {
    int nf = 0;
    for (int s = n_sink; s < P; ++s)
      if (holder[s] < 0) free_pos[nf++] = s;
  }
  __syncthreads();
  // newly kept blocks take free slots in ascending global-id order
  if (t < NI && it_rank[t] >= 0 && it_rank[t] < n_keep && it_old[t] < 0) {
    int r = 0;
    for (int u = 0; u < NI; ++u)
      if (it_rank[u] >= 0 && it_rank[u] < n_keep && it_old[u] < 0 && it_src[u] < it_src[t]) ++r;
    it_slot[t] = free_pos[r];
    holder[free_pos[r]] = t;
  }
  __syncthreads();

  // ---- merge targets: most similar kept slot by pooled-key dot product
  if (a.policy == PBSA_MERGE_MEAN && n_keep > 0) {
    for (int u = warp; u < NI; u += 8) {
      if (!(it_rank[u] >= n_keep)) continue;          // losers only (warp-uniform)
      const float* kj = a.k_bar + (bh * a.NB + it_phys[u]) * static_cast<long>(a.D);
      float best = -INFINITY;
      int best_s = -1;
      for (int s = n_sink; s < P; ++s) {
        const int c = holder[s];
        if (c < 0) continue;
        const float* kc = a.k_bar + (bh * a.NB + it_phys[c]) * static_cast<long>(a.D);
        float part = 0.f;
        for (int dd = lane; dd < a.D; dd += 32) part = fmaf(kj[dd], kc[dd], part);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        if (part > best || best_s < 0) { best = part; best_s = s; }
      }
      if (lane == 0) it_target[u] = best_s;
    }
  }
  __syncthreads();

  // ---- per-slot plan
  for (int s = t; s < P; s += 256) {
    int op = OP_NONE, base = -1, blen = 0, src = -1, pos = 0, stash = 0;
    float bw = 0.f;
    if (s < n_sink) {
      const int u = sink_item[s];
      if (u >= 0) {
        op = OP_WRITE; base = it_phys[u]; blen = it_len[u]; bw = 1.f; src = s;
        pos = a.blk_pos[bh * a.NB + base];
      }
    } else {
      const int c = holder[s];
      if (c < 0) {
        op = OP_CLEAR;
      } else {
        base = it_phys[c]; blen = it_len[c]; bw = it_w[c]; src = it_src[c];
        pos = a.blk_pos[bh * a.NB + base];
        bool merged = false;
        for (int u = 0; u < NI; ++u) merged |= (it_target[u] == s);
        op = (it_old[c] < 0 || merged) ? OP_WRITE : OP_NONE;
      }
    }
    pv.op[s] = op; pv.base[s] = base; pv.base_len[s] = blen; pv.base_w[s] = bw;
    pv.src[s] = src; pv.pos[s] = pos; pv.stash[s] = stash;
  }
  __syncthreads();
  // losers that are old slots overwritten by a new block are read from the stash
  if (t < NI && it_target[t] >= 0 && it_old[t] >= 0 && pv.op[it_old[t]] == OP_WRITE)
    pv.stash[it_old[t]] = 1;
  // merge lists grouped by target slot, each in ranking order (deterministic
  // summation order): counting sort over the losers
  __shared__ int tcount[256];
  for (int s = t; s < P; s += 256) tcount[s] = 0;
  __syncthreads();
  int my_pos = 0;
  const int my_target = (t < NI) ? it_target[t] : -1;
  if (my_target >= 0) {
    atomicAdd(&tcount[my_target], 1);
    for (int u = 0; u < NI; ++u)
      if (it_target[u] == my_target && it_rank[u] < it_rank[t]) ++my_pos;
  }
  __syncthreads();
  if (t == 0) {
    int off = 0;
    for (int s = 0; s < P; ++s) {
      pv.moff[s] = off;
      off += tcount[s];
    }
    pv.moff[P] = off;
  }
  __syncthreads();
  if (my_target >= 0) {
    const int slot = pv.moff[my_target] + my_pos;
    const int old = it_old[t];
    const bool from_stash = old >= 0 && pv.op[old] == OP_WRITE;
    pv.mref[slot] = from_stash ? -(1 + old) : it_phys[t];
    pv.mlen[slot] = it_len[t];
    pv.mw[slot] = it_w[t];
  }
}

// -------------------------------------------------------------------- stash
template <typename T>
__global__ void __launch_bounds__(256)
update_stash_kernel(UpdArgs a, const T* __restrict__ kpool, const T* __restrict__ vpool,
                    T* __restrict__ stash) {
  const int s = blockIdx.x;
  const long bh = blockIdx.y;
  PlanView pv = plan_view(a.ws, bh, a.P, a.M);
  if (!pv.stash[s]) return;
  const int n16 = static_cast<int>(static_cast<long>(a.bs) * a.D * sizeof(T) / 16);
  const uint4* ks = reinterpret_cast<const uint4*>(kpool + (bh * a.NB + s) * static_cast<long>(a.bs) * a.D);
  const uint4* vs = reinterpret_cast<const uint4*>(vpool + (bh * a.NB + s) * static_cast<long>(a.bs) * a.D);
  uint4* kd = reinterpret_cast<uint4*>(stash + ((bh * a.P + s) * 2 + 0) * static_cast<long>(a.bs) * a.D);
  uint4* vd = reinterpret_cast<uint4*>(stash + ((bh * a.P + s) * 2 + 1) * static_cast<long>(a.bs) * a.D);
  for (int e0 = 0; e0 < n16; e0 += 256 * 8) {
    uint4 ka[8], va[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int e = e0 + threadIdx.x + k * 256;
      if (e < n16) { ka[k] = ks[e]; va[k] = vs[e]; }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
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
  __device__ static void store(float* p, float (&x)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(256)
update_apply_kernel(UpdArgs a, T* __restrict__ kpool, T* __restrict__ vpool,
                    const T* __restrict__ stash, int32_t* __restrict__ blk_len,
                    int32_t* __restrict__ blk_pos, float* __restrict__ k_bar,
                    int32_t* __restrict__ slot_src, float* __restrict__ slot_w) {
  constexpr int EPC = Elem<T>::EPC;
  constexpr int CPR = D / EPC;
  constexpr int RPP = 256 / CPR;
  __shared__ float red[8][D];
  const int s = blockIdx.x;
  const long bh = blockIdx.y;
  const int t = threadIdx.x;
  PlanView pv = plan_view(a.ws, bh, a.P, a.M);
  const int op = pv.op[s];
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
  const int base = pv.base[s];
  const int m0 = pv.moff[s], m1 = pv.moff[s + 1];
  const int blen = pv.base_len[s];
  const float bw = pv.base_w[s];
  T* kd = kpool + (bh * a.NB + s) * blk_elems;
  T* vd = vpool + (bh * a.NB + s) * blk_elems;
  const T* kb = kpool + (bh * a.NB + base) * blk_elems;
  const T* vb = vpool + (bh * a.NB + base) * blk_elems;
  if (m0 == m1) {
    // plain copy of a newly admitted block (base != s)
    // source and destination are different blocks of the same pool: load a
    // batch of 16-byte chunks into registers, then store them
    const int n16 = static_cast<int>(blk_elems * sizeof(T) / 16);
    for (int e0 = 0; e0 < n16; e0 += 256 * 8) {
      uint4 ka[8], va[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int e = e0 + t + k * 256;
        if (e < n16) {
          ka[k] = reinterpret_cast<const uint4*>(kb)[e];
          va[k] = reinterpret_cast<const uint4*>(vb)[e];
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int e = e0 + t + k * 256;
        if (e < n16) {
          reinterpret_cast<uint4*>(kd)[e] = ka[k];
          reinterpret_cast<uint4*>(vd)[e] = va[k];
        }
      }
    }
    if (t < D) kb_out[t] = a.k_bar[(bh * a.NB + base) * static_cast<long>(D) + t];
    if (t == 0) {
      slot_src[bh * a.P + s] = pv.src[s];
      slot_w[bh * a.P + s] = bw;
      blk_len[bh * a.NB + s] = blen;
      blk_pos[bh * a.NB + s] = pv.pos[s];
    }
    return;
  }
  // weighted row-wise mean of the base and its merged losers
  float wsum = bw;
  int nlen = blen;
  for (int m = m0; m < m1; ++m) {
    wsum += pv.mw[m];
    nlen = max(nlen, pv.mlen[m]);
  }
  const float inv = 1.f / wsum;
  const int c = t % CPR, rg = t / CPR;
  float colsum[EPC];
#pragma unroll
  for (int e = 0; e < EPC; ++e) colsum[e] = 0.f;
  for (int r = rg; r < a.bs; r += RPP) {
    const long off = static_cast<long>(r) * D + c * EPC;
    float ak[EPC], av[EPC], x[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) { ak[e] = 0.f; av[e] = 0.f; }
    if (r < blen) {
      Elem<T>::load(kb + off, x);
#pragma unroll
      for (int e = 0; e < EPC; ++e) ak[e] = bw * x[e];
      Elem<T>::load(vb + off, x);
#pragma unroll
      for (int e = 0; e < EPC; ++e) av[e] = bw * x[e];
    }
    for (int m = m0; m < m1; ++m) {
      if (r >= pv.mlen[m]) continue;
      const int ref = pv.mref[m];
      const float w = pv.mw[m];
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
      Elem<T>::load(ks + off, x);
#pragma unroll
      for (int e = 0; e < EPC; ++e) ak[e] = fmaf(w, x[e], ak[e]);
      Elem<T>::load(vs + off, x);
#pragma unroll
      for (int e = 0; e < EPC; ++e) av[e] = fmaf(w, x[e], av[e]);
    }
#pragma unroll
    for (int e = 0; e < EPC; ++e) { ak[e] *= inv; av[e] *= inv; }
    // every thread reads its own elements above before writing them here
    Elem<T>::store(kd + off, ak);
    Elem<T>::store(vd + off, av);
    if (r < nlen) {
#pragma unroll
      for (int e = 0; e < EPC; ++e) colsum[e] += ak[e];
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
    slot_src[bh * a.P + s] = pv.src[s];
    slot_w[bh * a.P + s] = wsum;
    blk_len[bh * a.NB + s] = nlen;
    blk_pos[bh * a.NB + s] = pv.pos[s];
  }
}

size_t stash_bytes(const pbsa_dims* d, int P) {
  return align_up(static_cast<size_t>(d->B) * d->H * P * 2 * d->bs * d->D * elem_size(d->dtype),
                  256);
}

template <typename T, int D>
void launch_apply(const UpdArgs& a, void* kpool, void* vpool, const void* stash, int32_t* blk_len,
                  int32_t* blk_pos, float* k_bar, int32_t* slot_src, float* slot_w,
                  cudaStream_t s) {
  dim3 grid(a.P, a.B * a.H);
  if (a.policy == PBSA_MERGE_MEAN)
    update_stash_kernel<T><<<grid, 256, 0, s>>>(a, static_cast<const T*>(kpool),
                                                static_cast<const T*>(vpool),
                                                static_cast<T*>(const_cast<void*>(stash)));
  update_apply_kernel<T, D><<<grid, 256, 0, s>>>(a, static_cast<T*>(kpool), static_cast<T*>(vpool),
                                                 static_cast<const T*>(stash), blk_len, blk_pos,
                                                 k_bar, slot_src, slot_w);
}

}  // namespace
}  // namespace pbsa

extern "C" size_t pbsa_update_memory_workspace(const pbsa_dims* d, int P, int n_cand) {
  using namespace pbsa;
  if (d == nullptr || P < 1 || n_cand < 0 || d->B < 1 || d->H < 1) return 0;
  const int M = P + n_cand;
  return static_cast<size_t>(d->B) * d->H * plan_bytes(P, M) + stash_bytes(d, P);
}

extern "C" int pbsa_update_memory(const pbsa_dims* d, void* kpool, void* vpool, int NB,
                                  int32_t* blk_len, int32_t* blk_pos, float* k_bar, int P,
                                  int n_sink, int32_t* slot_src, float* slot_w,
                                  const int32_t* cand_ids, const int32_t* cand_src, int n_cand,
                                  const float* mem_score, int policy, void* workspace,
                                  size_t ws_bytes, void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(kpool && vpool && blk_len && blk_pos && k_bar && slot_src && slot_w && mem_score,
                 PBSA_ERR_ARG, "update_memory: NULL buffer");
  PBSA_CHECK_ARG(n_cand >= 0 && (n_cand == 0 || (cand_ids && cand_src)), PBSA_ERR_ARG,
                 "update_memory: candidate lists are NULL");
  PBSA_CHECK_ARG(P >= 1 && P <= 256 && NB >= P, PBSA_ERR_SHAPE,
                 "update_memory: need 1 <= P <= 256 and NB >= P");
  PBSA_CHECK_ARG(n_sink >= 0 && n_sink <= P, PBSA_ERR_SHAPE, "update_memory: bad n_sink");
  PBSA_CHECK_ARG((P - n_sink) + n_cand <= kMaxItems, PBSA_ERR_SHAPE,
                 "update_memory: (P - n_sink) + n_cand must be <= 256");
  PBSA_CHECK_ARG(policy == PBSA_EVICT || policy == PBSA_MERGE_MEAN, PBSA_ERR_ARG,
                 "update_memory: bad policy");
  PBSA_CHECK_ARG(aligned(kpool, 16) && aligned(vpool, 16), PBSA_ERR_ALIGN,
                 "update_memory: kpool/vpool must be 16-byte aligned");
  PBSA_CHECK_ARG(static_cast<long>(d->B) * d->H <= 65535, PBSA_ERR_SHAPE,
                 "update_memory: B*H must be <= 65535");
  const size_t need = pbsa_update_memory_workspace(d, P, n_cand);
  PBSA_CHECK_ARG(workspace != nullptr && ws_bytes >= need && aligned(workspace, 256),
                 PBSA_ERR_WORKSPACE,
                 "update_memory: workspace missing, too small or not 256-byte aligned (need " +
                     std::to_string(need) + " bytes)");
  int* status = device_status_ptr();
  PBSA_CHECK_ARG(status != nullptr, PBSA_ERR_CUDA, "update_memory: no device status word");
  UpdArgs a;
  a.B = d->B; a.H = d->H; a.D = d->D; a.bs = d->bs; a.NB = NB; a.P = P; a.n_sink = n_sink;
  a.n_cand = n_cand; a.policy = policy; a.M = P + n_cand;
  a.blk_len = blk_len; a.blk_pos = blk_pos; a.k_bar = k_bar; a.slot_src = slot_src;
  a.slot_w = slot_w; a.cand_ids = cand_ids; a.cand_src = cand_src; a.mem = mem_score;
  a.ws = workspace; a.status = status;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  update_plan_kernel<<<d->B * d->H, 256, 0, s>>>(a);
  PBSA_CHECK_LAUNCH("update_plan_kernel");
  const void* stash =
      static_cast<const char*>(workspace) + static_cast<size_t>(d->B) * d->H * plan_bytes(P, a.M);
  if (d->dtype == PBSA_BF16) {
    if (d->D == 128)
      launch_apply<__nv_bfloat16, 128>(a, kpool, vpool, stash, blk_len, blk_pos, k_bar, slot_src,
                                       slot_w, s);
    else
      launch_apply<__nv_bfloat16, 64>(a, kpool, vpool, stash, blk_len, blk_pos, k_bar, slot_src,
                                      slot_w, s);
  } else {
    if (d->D == 128)
      launch_apply<float, 128>(a, kpool, vpool, stash, blk_len, blk_pos, k_bar, slot_src, slot_w,
                               s);
    else
      launch_apply<float, 64>(a, kpool, vpool, stash, blk_len, blk_pos, k_bar, slot_src, slot_w, s);
  }
  PBSA_CHECK_LAUNCH("update_apply_kernel");
  return PBSA_OK;
}
