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
// score_item: one (b,h, 16 key blocks) item.  Each thread keeps half of one
// pooled key in registers; the query-block means are staged in shared memory;
// S is written row by row and the memory score of every query chunk (the mean
// of S over the chunk's query blocks, summed in block order) is formed from a
// shared-memory copy of the item's S columns.
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

constexpr int kScoreJ = 16;     // key blocks per CTA
constexpr int kScoreQI = 64;    // query blocks staged per pass
constexpr int kScoreTileMax = 1024;   // query blocks whose S columns stay in shared memory

struct ScoreArgs {
  const float* q_bar;
  const float* k_bar;
  float* scores;
  float* mem;
  int nQB, NB, per_group, groups;
  float scale;
};

// Scores of key blocks [16 jblk, 16 jblk + 16) against every query block of
// head bh, and their memory scores.  `ssm` holds score_smem_bytes() bytes.
template <int D>
__device__ void score_item(const ScoreArgs& a, long bh, int jblk, float* ssm) {
  const int QI = min(a.nQB, kScoreQI);
  float4* qs = reinterpret_cast<float4*>(ssm);            // [QI][D/4]
  float* st = ssm + QI * D;                               // [nQB][16] when kept
  const bool keep = a.nQB <= kScoreTileMax;
  const int j0 = jblk * kScoreJ;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int jj = lane & 15, half = lane >> 4;
  const int j = j0 + jj;
  // half `half` of pooled key j: float4 number 2m + half, m < D/8
  constexpr int NV = D / 8;
  float4 kr[NV];
  {
    const float4* krow =
        reinterpret_cast<const float4*>(a.k_bar + (bh * a.NB + min(j, a.NB - 1)) * D);
#pragma unroll
    for (int m = 0; m < NV; ++m) kr[m] = krow[2 * m + half];
  }
  const float4* qsrc = reinterpret_cast<const float4*>(a.q_bar + bh * a.nQB * D);
  for (int i0 = 0; i0 < a.nQB; i0 += QI) {
    const int ni = min(QI, a.nQB - i0);
    __syncthreads();
    // all of a thread's loads in flight together (8 per batch)
    for (int e0 = 0; e0 < ni * (D / 4); e0 += 256 * 8) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = e0 + u * 256 + t;
        if (e < ni * (D / 4)) v[u] = qsrc[i0 * (D / 4) + e];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = e0 + u * 256 + t;
        if (e < ni * (D / 4)) qs[e] = v[u];
      }
    }
    __syncthreads();
    for (int ii = warp; ii < ni; ii += 8) {
      const float4* qr = qs + ii * (D / 4);
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int m = 0; m < NV; ++m) {
        const float4 q = qr[2 * m + half];
        s0 = fmaf(q.x, kr[m].x, s0);
        s1 = fmaf(q.y, kr[m].y, s1);
        s0 = fmaf(q.z, kr[m].z, s0);
        s1 = fmaf(q.w, kr[m].w, s1);
      }
      float s = s0 + s1;
      s += __shfl_xor_sync(0xffffffffu, s, 16);
      s *= a.scale;
      if (half == 0 && j < a.NB) {
        a.scores[(bh * a.nQB + i0 + ii) * a.NB + j] = s;
        if (keep) st[(i0 + ii) * kScoreJ + jj] = s;
      }
    }
  }
  __syncthreads();
  // memory score of every query chunk: mean of S over its query blocks, in
  // block order
  for (int e = t; e < a.groups * kScoreJ; e += 256) {
    const int g = e / kScoreJ, c = e % kScoreJ, jc = j0 + c;
    if (jc >= a.NB) continue;
    const int i_lo = g * a.per_group, i_hi = min(a.nQB, (g + 1) * a.per_group);
    float m = 0.f;
    if (keep) {
      for (int i = i_lo; i < i_hi; ++i) m += st[i * kScoreJ + c];
    } else {
      for (int i = i_lo; i < i_hi; ++i) m += a.scores[(bh * a.nQB + i) * a.NB + jc];
    }
    a.mem[(bh * a.groups + g) * a.NB + jc] = m / static_cast<float>(i_hi - i_lo);
  }
}

template <int D>
__host__ __device__ inline size_t score_smem_bytes(int nQB) {
  const int QI = nQB < kScoreQI ? nQB : kScoreQI;
  return static_cast<size_t>(QI) * D * sizeof(float) +
         (nQB <= kScoreTileMax ? static_cast<size_t>(nQB) * kScoreJ * 4 : 0);
}

}  // namespace dev
}  // namespace pbsa
