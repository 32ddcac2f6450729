// Device code of a1 + a2 (block pooling and coarse block scoring), shared by
// the per-call kernels (pool_score.cu) and the fused routing kernel (route.cu).
//
// Sparse Forcing compresses each spatiotemporal block into a pooled
// representative for cheap, coarse routing (gist.science/es, section 2,
// PBSA item "Compresión de Bloques") and scores historical blocks for their
// relevance to the current step (item "Bloques Dinámicos").
//
// pool_phase (HBM-bound): a CTA walks its share of the blocks to pool (query
// blocks and the listed key blocks).  Each block is one contiguous run of
// rows, brought into a ring of shared-memory stages by an untiled bulk copy
// (cp.async.bulk, completion on an mbarrier), so every CTA keeps several whole
// blocks in flight; the rows are summed in fp32 from shared memory with
// 128-bit reads and a warp-shuffle + shared-memory reduction.  Every input
// byte is read once.
// score_item: one square tile of S (b,h, T query blocks x T key blocks) as a
// small fp32 GEMM on the CUDA cores, from q_bar / k_bar rows staged by cp.async;
// the memory scores of the query chunks that start in the tile come from the
// chunk's mean pooled query, so tiles are independent of one another.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "tc_sm100.cuh"

namespace pbsa {
namespace dev {

using namespace tc;

constexpr int kPoolThreads = 256;
constexpr int kPoolCtasPerSm = 2;
constexpr int kPoolStageBudget = 96 * 1024;   // shared memory for stages per CTA
constexpr int kPoolMeta = 32;                 // items whose addresses are looked up up front

struct PoolArgs {
  const void* q;
  const void* kpool;
  const int32_t* blk_len;
  const int32_t* pool_ids;
  float* q_bar;
  float* k_bar;
  int Tq, qc, NB, bs, nQB, n_pool, n_items, stages;
  int* status;
  int64_t limit_ns;
};

template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int EPC = 8;
  __device__ static void add(const uint8_t* p, float (&acc)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    acc[0] += bf16_lo(u.x); acc[1] += bf16_hi(u.x);
    acc[2] += bf16_lo(u.y); acc[3] += bf16_hi(u.y);
    acc[4] += bf16_lo(u.z); acc[5] += bf16_hi(u.z);
    acc[6] += bf16_lo(u.w); acc[7] += bf16_hi(u.w);
  }
};
template <>
struct Vec16<float> {
  static constexpr int EPC = 4;
  __device__ static void add(const uint8_t* p, float (&acc)[4]) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    acc[0] += u.x; acc[1] += u.y; acc[2] += u.z; acc[3] += u.w;
  }
};

// Column sums of rows [0, n) of a block staged in shared memory (rows of D
// elements of T, 16-byte chunks), reduced to one partial row per warp in
// rb[8][D].  Every thread of the 256-thread CTA calls it; the caller
// synchronises before row_mean() reads rb.  Shared by the pooling of
// pbsa_score_blocks and pbsa_append_chunk, so both give the same means.
template <typename T, int D>
__device__ __forceinline__ void row_sums(const uint8_t* stage, int n, float* rb) {
  constexpr int EPC = Vec16<T>::EPC;
  constexpr int CPR = D / EPC;
  constexpr int RPP = kPoolThreads / CPR;
  constexpr int ROW = D * static_cast<int>(sizeof(T));
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int c = t % CPR, rg = t / CPR;
  float acc[EPC];
#pragma unroll
  for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
#pragma unroll 4
  for (int r = rg; r < n; r += RPP) Vec16<T>::add(stage + r * ROW + c * 16, acc);
#pragma unroll
  for (int off = CPR; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  if (lane < CPR) {
#pragma unroll
    for (int e = 0; e < EPC; ++e) rb[warp * D + lane * EPC + e] = acc[e];
  }
}

// Mean of column t (t < D) from the per-warp partial rows.
template <int D>
__device__ __forceinline__ float row_mean(const float* rb, int n) {
  const int t = threadIdx.x;
  float sum = 0.f;
#pragma unroll
  for (int w = 0; w < kPoolThreads / 32; ++w) sum += rb[w * D + t];
  return n > 0 ? sum / static_cast<float>(n) : 0.f;
}

// Where item `it` (flattened over (b,h) x [query blocks, listed key blocks])
// reads its rows and where its mean goes: `out` >= 0 is an offset into q_bar,
// `out` <= -2 is the offset -(out + 2) into k_bar, -1 means no output (an
// invalid id).  n = number of valid rows (0: nothing to copy, the mean is 0).
template <typename T, int D>
__device__ __forceinline__ void pool_item(const PoolArgs& a, int it, const T*& src, long& out,
                                          int& n) {
  const int per = a.nQB + a.n_pool;
  const long bh = it / per;
  const int item = it - static_cast<int>(bh) * per;
  if (item < a.nQB) {
    int row0;
    qb_rows(item, a.Tq, a.qc, a.bs, row0, n);
    src = static_cast<const T*>(a.q) + (bh * a.Tq + row0) * static_cast<long>(D);
    out = (bh * a.nQB + item) * D;
  } else {
    const int id = a.pool_ids[item - a.nQB];
    if (id < 0 || id >= a.NB) {
      report_status(a.status, PBSA_ERR_ARG);
      src = nullptr;
      out = -1;
      n = 0;
      return;
    }
    n = min(max(a.blk_len[bh * a.NB + id], 0), a.bs);
    src = static_cast<const T*>(a.kpool) + (bh * a.NB + id) * static_cast<long>(a.bs) * D;
    out = -(2 + (bh * a.NB + id) * D);
  }
}

// Pool every item of this CTA's share (items cta, cta + G, ...).  `smem` holds
// pool_smem_bytes() bytes.  The mbarriers it uses are invalidated on the way
// out, so the caller may reuse the memory.
template <typename T, int D>
__device__ void pool_phase(const PoolArgs& a, int cta, int G, uint8_t* smem) {
  constexpr int EPC = Vec16<T>::EPC;
  constexpr int CPR = D / EPC;                 // 16-byte chunks per row
  constexpr int ROW = D * static_cast<int>(sizeof(T));
  static_assert(CPR <= 32 && (32 % CPR) == 0, "chunks per row must divide a warp");
  const int S = a.stages;
  const int stage_bytes = a.bs * ROW;
  float* red = reinterpret_cast<float*>(smem + S * stage_bytes);        // [2][8][D]
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 2 * 8 * D);         // [S]
  long* s_out = reinterpret_cast<long*>(bars + S);                       // [S] out offset or -1
  const T** m_src = reinterpret_cast<const T**>(s_out + S);              // [kPoolMeta]
  long* m_out = reinterpret_cast<long*>(m_src + kPoolMeta);              // [kPoolMeta]
  int* s_n = reinterpret_cast<int*>(m_out + kPoolMeta);                  // [S]
  int* m_n = s_n + S;                                                    // [kPoolMeta]
  volatile int* abort_flag = m_n + kPoolMeta;

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int mine = a.n_items > cta ? (a.n_items - cta + G - 1) / G : 0;
  if (t == 0) {
    for (int s = 0; s < S; ++s) mbar_init(smem_u32(&bars[s]), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // where the CTA's first kPoolMeta items read and write, looked up by the
  // lanes of warp 0 at once (each lookup is a chain of dependent loads)
  if (warp == 0) {
    for (int k = lane; k < min(mine, kPoolMeta); k += 32) {
      const T* src;
      long out;
      int n;
      pool_item<T, D>(a, cta + k * G, src, out, n);
      m_src[k] = src;
      m_out[k] = out;
      m_n[k] = n;
    }
    __syncwarp();
  }

  // thread 0 issues item k of this CTA into stage k % S
  auto issue = [&](int k) {
    const int s = k % S;
    const T* src;
    long out;
    int n;
    if (k < kPoolMeta) {
      src = m_src[k];
      out = m_out[k];
      n = m_n[k];
    } else {
      pool_item<T, D>(a, cta + k * G, src, out, n);
    }
    s_n[s] = n;
    s_out[s] = out;
    const uint32_t bar = smem_u32(&bars[s]);
    if (n > 0) {
      mbar_expect_tx(bar, static_cast<uint32_t>(n * ROW));
      bulk_load(smem_u32(smem + s * stage_bytes), src, static_cast<uint32_t>(n * ROW), bar);
    } else {
      mbar_arrive(bar);
    }
  };

  int issued = 0;
  if (t == 0) {
    const int first = min(S, mine);
    for (int k = 0; k < first; ++k) issue(k);
    issued = first;
  }
  bool ok = true;
  for (int k = 0; k < mine; ++k) {
    const int s = k % S;
    ok = mbar_wait(smem_u32(&bars[s]), static_cast<uint32_t>((k / S) & 1), abort_flag, a.status,
                   a.limit_ns);
    if (__syncthreads_or(!ok)) { ok = false; break; }
    const int n = s_n[s];
    const long oo = s_out[s];
    float* rb = red + (k & 1) * 8 * D;
    row_sums<T, D>(smem + s * stage_bytes, n, rb);
    __syncthreads();   // stage s fully read; partial sums of item k complete
    if (t == 0 && k + S < mine) {
      issue(k + S);
      ++issued;
    }
    if (t < D && oo != -1) {
      float* out = oo >= 0 ? a.q_bar + oo : a.k_bar + (-(oo + 2));
      out[t] = row_mean<D>(rb, n);
    }
  }
  // on a time-out, wait for the copies still in flight before the CTA exits:
  // the last S issued items cover every stage; a phase that already completed
  // passes at once
  if (t == 0 && !ok) {
    for (int k = max(0, issued - S); k < issued; ++k)
      mbar_drain(smem_u32(&bars[k % S]), static_cast<uint32_t>((k / S) & 1), a.status,
                 a.limit_ns);
  }
  __syncthreads();
  if (t < S) mbar_inval(smem_u32(&bars[t]));
  __syncthreads();
}

template <typename T, int D>
__host__ __device__ inline size_t pool_smem_bytes(int stages, int bs) {
  return static_cast<size_t>(stages) * bs * D * sizeof(T) + 2 * 8 * D * sizeof(float) +
         stages * (sizeof(uint64_t) + sizeof(long) + sizeof(int)) +
         kPoolMeta * (sizeof(void*) + sizeof(long) + sizeof(int)) + 16;
}

template <typename T, int D>
__host__ __device__ inline int pool_stages(int bs) {
  const int stage_bytes = bs * D * static_cast<int>(sizeof(T));
  const int st = kPoolStageBudget / stage_bytes;
  return st < 2 ? 2 : (st > 4 ? 4 : st);
}

// Tiles of S: the per-call scoring kernel runs 32 x 32 tiles on 64-thread
// CTAs, 4 x 4 scores per thread (enough CTAs to cover the SMs on a decode
// step's few hundred tiles); the fused routing kernel runs 32 x 32 tiles on its
// 256 threads, 2 x 2 scores per thread, so a head's scores spread over more
// SMs.  Every score and memory score is computed in the same order in both, so
// the two give the same bits.
constexpr int kScoreTile = 32, kScoreThreads = 64;
constexpr int kRouteScoreTile = 32;

struct ScoreArgs {
  const float* q_bar;
  const float* k_bar;
  float* scores;
  float* mem;
  int nQB, NB, per_group, groups;
  float scale;
};

// Row pitch (floats) of the staged q_bar / k_bar tiles: D + 4 puts the 8
// rows a quarter-warp reads at once on distinct bank groups.
template <int D>
__host__ __device__ constexpr int score_pitch() { return D + 4; }

// Stage rows [0, n) of a [*, D] fp32 matrix as the TR rows of a padded tile
// (NT threads): 16-byte asynchronous copies (cp.async, no registers held, all
// of a thread's copies in flight at once), zeros for rows past n.  The caller
// waits with score_stage_wait() and then synchronises the CTA.
template <int D, int TR, int NT>
__device__ __forceinline__ void score_stage(float* tile, const float* src, int n) {
  constexpr int PER = TR * (D / 4) / NT;
  static_assert(PER * NT == TR * (D / 4), "tile must split evenly over the threads");
  const int t = threadIdx.x;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int e = t + u * NT, row = e / (D / 4), c4 = e % (D / 4);
    float* dst = tile + row * score_pitch<D>() + c4 * 4;
    if (row < n) {
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst)),
                   "l"(src + static_cast<long>(e) * 4)
                   : "memory");
    } else {
      *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}
__device__ __forceinline__ void score_stage_wait() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

// <qm, k> of one key row, split over the four lanes of a quad (lane p takes
// the float4 numbers p + 4m, one fmaf chain each) and combined as
// (s0 + s1) + (s2 + s3).  All four lanes of the quad call it and get the sum.
// Every memory score of the library is this function times the scale.
template <int D>
__device__ __forceinline__ float quad_dot(const float* qm, const float* k, int p) {
  float s = 0.f;
#pragma unroll
  for (int m = 0; m < D / 16; ++m) {
    const float4 x = *reinterpret_cast<const float4*>(qm + (p + 4 * m) * 4);
    const float4 y = *reinterpret_cast<const float4*>(k + (p + 4 * m) * 4);
    s = fmaf(x.x, y.x, s);
    s = fmaf(x.y, y.y, s);
    s = fmaf(x.z, y.z, s);
    s = fmaf(x.w, y.w, s);
  }
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  return s;
}

// One T x T tile of S: query blocks [T itile, +T) against key blocks
// [T jblk, +T) of head bh, plus the memory scores of the query chunks that
// start inside the tile's rows.  Called by all NT = (T/R)^2 threads of the CTA.
//
// The tile is a small fp32 GEMM on the CUDA cores (K = D is short, and the
// scores are compared against a selection threshold, so no reduced-precision
// tensor-core inputs): thread (ty, tx) of the (T/R) x (T/R) grid owns rows
// ty + (T/R) k and columns tx + (T/R) l (k, l < R); every score is one fmaf
// chain over d = 0 .. D-1 in order, times scale.
//
// The memory score of chunk g is the mean of its scores over its query blocks.
// The scores are linear in the pooled query, so that mean is computed as
// scale * <mean of the chunk's pooled queries, k_bar_j> (equal up to rounding):
// the chunk's mean query (sum in block order, fp32, then one divide), then one
// quad_dot per key block.  The tile holding the chunk's first query block does
// it, so no tile waits on another.
template <int D, int T, int R = 4>
__device__ void score_item(const ScoreArgs& a, long bh, int jblk, int itile, float* ssm) {
  constexpr int PT = score_pitch<D>();
  constexpr int GR = T / R, NT = GR * GR;
  float* ks = ssm;                                         // [T][PT]
  float* qs = ks + T * PT;                                 // [T][PT]
  float* qm = qs + T * PT;                                 // [D] a chunk's mean query
  const int t = threadIdx.x, tx = t % GR, ty = t / GR;
  const int j0 = jblk * T, i0 = itile * T;
  const int nj = min(T, a.NB - j0), ni = min(T, a.nQB - i0);
  const float* qrows = a.q_bar + bh * a.nQB * D;
  __syncthreads();                    // the previous item's readers are done
  score_stage<D, T, NT>(ks, a.k_bar + (bh * a.NB + j0) * D, nj);
  score_stage<D, T, NT>(qs, qrows + static_cast<long>(i0) * D, ni);
  score_stage_wait();
  __syncthreads();
  float acc[R][R];
#pragma unroll
  for (int k = 0; k < R; ++k)
#pragma unroll
    for (int l = 0; l < R; ++l) acc[k][l] = 0.f;
#pragma unroll 4
  for (int d = 0; d < D; d += 4) {
    float4 q[R], kk[R];
#pragma unroll
    for (int k = 0; k < R; ++k) q[k] = *reinterpret_cast<const float4*>(qs + (ty + GR * k) * PT + d);
#pragma unroll
    for (int l = 0; l < R; ++l) kk[l] = *reinterpret_cast<const float4*>(ks + (tx + GR * l) * PT + d);
#pragma unroll
    for (int k = 0; k < R; ++k)
#pragma unroll
      for (int l = 0; l < R; ++l) {
        float s = acc[k][l];
        s = fmaf(q[k].x, kk[l].x, s);
        s = fmaf(q[k].y, kk[l].y, s);
        s = fmaf(q[k].z, kk[l].z, s);
        s = fmaf(q[k].w, kk[l].w, s);
        acc[k][l] = s;
      }
  }
#pragma unroll
  for (int k = 0; k < R; ++k) {
    const int r = ty + GR * k;
#pragma unroll
    for (int l = 0; l < R; ++l) {
      const int c = tx + GR * l;
      if (r < ni && c < nj) a.scores[(bh * a.nQB + i0 + r) * a.NB + j0 + c] = acc[k][l] * a.scale;
    }
  }
  // chunks whose first query block is in rows [i0, i0 + ni)
  const int g_lo = (i0 + a.per_group - 1) / a.per_group;
  const int g_hi = min(a.groups, (i0 + ni + a.per_group - 1) / a.per_group);
  for (int g = g_lo; g < g_hi; ++g) {
    const int r_lo = g * a.per_group, r_hi = min(a.nQB, r_lo + a.per_group);
    const int r_mid = min(r_hi, i0 + ni);          // rows below r_mid are staged
    {
      // the DPT columns of a thread summed side by side, so the rows past the
      // staged tile cost one round of loads, not DPT
      constexpr int DPT = (D + NT - 1) / NT;
      float sum[DPT];
#pragma unroll
      for (int u = 0; u < DPT; ++u) sum[u] = 0.f;
      for (int i = r_lo; i < r_mid; ++i) {
#pragma unroll
        for (int u = 0; u < DPT; ++u)
          if (t + u * NT < D) sum[u] += qs[(i - i0) * PT + t + u * NT];
      }
#pragma unroll 8
      for (int i = r_mid; i < r_hi; ++i) {
#pragma unroll
        for (int u = 0; u < DPT; ++u)
          if (t + u * NT < D) sum[u] += qrows[static_cast<long>(i) * D + t + u * NT];
      }
#pragma unroll
      for (int u = 0; u < DPT; ++u)
        if (t + u * NT < D) qm[t + u * NT] = sum[u] / static_cast<float>(r_hi - r_lo);
    }
    __syncthreads();
    const int p = t & 3;
    for (int c = t >> 2; c < T; c += NT / 4) {
      const float s = quad_dot<D>(qm, ks + c * PT, p);
      if (p == 0 && c < nj) a.mem[(bh * a.groups + g) * a.NB + j0 + c] = s * a.scale;
    }
    __syncthreads();                  // qm free for the next chunk
  }
}

template <int D, int T>
__host__ __device__ inline size_t score_smem_bytes() {
  return static_cast<size_t>(2 * T * score_pitch<D>() + D) * sizeof(float);
}

}  // namespace dev
}  // namespace pbsa
