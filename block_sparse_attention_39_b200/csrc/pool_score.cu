// a1 + a2: block pooling and coarse block scoring.
//
// Sparse Forcing compresses each spatiotemporal block into a pooled
// representative for cheap, coarse routing (gist.science/es, section 2,
// PBSA item "Compresión de Bloques") and scores historical blocks for their
// relevance to the current step (item "Bloques Dinámicos").
//
// Kernel 1 (pool): one CTA per block to pool (query blocks and the listed key
// blocks), 128-bit loads, fp32 accumulation, warp-shuffle + shared-memory
// reduction.  HBM-bound: every input byte is read once.
// Kernel 2 (score): one CTA per (b,h, 32 key blocks); the query-block means
// are staged in shared memory; writes S and the memory score of every query
// chunk (the mean of S over the chunk's query blocks).
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace pbsa {
namespace {

constexpr int kPoolThreads = 256;

template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int EPC = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&x)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x);
    x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
    x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z);
    x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
  }
};
template <>
struct Vec16<float> {
  static constexpr int EPC = 4;
  __device__ static void load(const float* p, float (&x)[4]) {
    float4 u = __ldg(reinterpret_cast<const float4*>(p));
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(kPoolThreads)
pool_kernel(const T* __restrict__ q, int Tq, int qc, const T* __restrict__ kpool, int NB, int bs,
            const int32_t* __restrict__ blk_len, const int32_t* __restrict__ pool_ids, int nQB,
            float* __restrict__ q_bar, float* __restrict__ k_bar, int* status) {
  constexpr int EPC = Vec16<T>::EPC;
  constexpr int CPR = D / EPC;                 // 16-byte chunks per row
  constexpr int RPP = kPoolThreads / CPR;      // rows per pass
  static_assert(CPR <= 32 && (32 % CPR) == 0, "chunks per row must divide a warp");
  __shared__ float red[kPoolThreads / 32][D];

  const int item = blockIdx.x;
  const long bh = blockIdx.y;
  const T* base;
  float* out;
  int n;
  if (item < nQB) {
    int row0;
    qb_rows(item, Tq, qc, bs, row0, n);
    base = q + (bh * Tq + row0) * static_cast<long>(D);
    out = q_bar + (bh * nQB + item) * D;
  } else {
    const int id = pool_ids[item - nQB];
    if (id < 0 || id >= NB) {
      if (threadIdx.x == 0) report_status(status, PBSA_ERR_ARG);
      return;
    }
    n = blk_len[bh * NB + id];
    n = max(0, min(n, bs));
    base = kpool + ((bh * NB + id) * static_cast<long>(bs)) * D;
    out = k_bar + (bh * NB + id) * D;
  }

  const int t = threadIdx.x;
  const int c = t % CPR;
  const int rg = t / CPR;
  float acc[EPC];
#pragma unroll
  for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
  // a block has at most 128 rows: at most 128 / RPP loads per thread, all in flight together
  constexpr int MAXR = (128 + RPP - 1) / RPP;
  float x[MAXR][EPC];
#pragma unroll
  for (int k = 0; k < MAXR; ++k) {
    const int r = rg + k * RPP;
    if (r < n) {
      Vec16<T>::load(base + static_cast<long>(r) * D + c * EPC, x[k]);
    } else {
#pragma unroll
      for (int e = 0; e < EPC; ++e) x[k][e] = 0.f;
    }
  }
#pragma unroll
  for (int k = 0; k < MAXR; ++k)
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] += x[k][e];
  // lanes l and l ^ (CPR * 2^k) hold the same chunk
#pragma unroll
  for (int off = CPR; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  const int lane = t & 31, warp = t >> 5;
  if (lane < CPR) {
#pragma unroll
    for (int e = 0; e < EPC; ++e) red[warp][lane * EPC + e] = acc[e];
  }
  __syncthreads();
  if (t < D) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kPoolThreads / 32; ++w) s += red[w][t];
    out[t] = n > 0 ? s / static_cast<float>(n) : 0.f;
  }
}

constexpr int kScoreJ = 32;   // key blocks per CTA (one per lane)
constexpr int kScoreI = 32;   // query blocks staged per pass (static smem < 48 KB)

template <int D>
__global__ void __launch_bounds__(256)
score_kernel(const float* __restrict__ q_bar, const float* __restrict__ k_bar, int nQB, int NB,
             float scale, float* __restrict__ scores, float* __restrict__ mem, int per_group,
             int groups) {
  __shared__ float kb[kScoreJ][D + 1];
  __shared__ __align__(16) float qb[kScoreI][D];
  const long bh = blockIdx.y;
  const int j0 = blockIdx.x * kScoreJ;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  {
    // 32 x D floats as float4: (8 * D / 256) loads per thread, issued together
    constexpr int NV = kScoreJ * D / 4 / 256;
    float4 v[NV];
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int e = (t + k * 256) * 4;
      const int jj = e / D;
      v[k] = (j0 + jj < NB) ? *reinterpret_cast<const float4*>(k_bar + (bh * NB + j0 + jj) * D + e % D)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int e = (t + k * 256) * 4;
      float* dst = &kb[e / D][e % D];
      dst[0] = v[k].x; dst[1] = v[k].y; dst[2] = v[k].z; dst[3] = v[k].w;
    }
  }
  const int j = j0 + lane;
  for (int i0 = 0; i0 < nQB; i0 += kScoreI) {
    const int ni = min(kScoreI, nQB - i0);
    __syncthreads();
    {
      constexpr int NV = kScoreI * D / 4 / 256;
      float4 v[NV];
      const float4* src = reinterpret_cast<const float4*>(q_bar + (bh * nQB + i0) * D);
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int e4 = t + k * 256;
        v[k] = (e4 * 4 < ni * D) ? src[e4] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int k = 0; k < NV; ++k) reinterpret_cast<float4*>(&qb[0][0])[t + k * 256] = v[k];
    }
    __syncthreads();
    for (int ii = warp; ii < ni; ii += 8) {
      float s = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) s = fmaf(qb[ii][d], kb[lane][d], s);
      if (j < NB) scores[(bh * nQB + i0 + ii) * NB + j] = s * scale;
    }
  }
  // memory score: mean over the query blocks of each query chunk, summed in
  // block order from the scores this CTA just wrote
  __syncthreads();
  for (int e = t; e < groups * kScoreJ; e += 256) {
    const int g = e / kScoreJ, jj = j0 + e % kScoreJ;
    if (jj >= NB) continue;
    const int i_lo = g * per_group, i_hi = min(nQB, (g + 1) * per_group);
    float m = 0.f;
    for (int i = i_lo; i < i_hi; ++i) m += scores[(bh * nQB + i) * NB + jj];
    mem[(bh * groups + g) * NB + jj] = m / static_cast<float>(i_hi - i_lo);
  }
}

template <typename T, int D>
void launch_pool(const pbsa_dims* d, const void* q, int Tq, const void* kpool, int NB,
                 const int32_t* blk_len, const int32_t* pool_ids, int n_pool, int nQB,
                 float* q_bar, float* k_bar, int* status, cudaStream_t s) {
  dim3 grid(nQB + n_pool, d->B * d->H);
  pool_kernel<T, D><<<grid, kPoolThreads, 0, s>>>(
      static_cast<const T*>(q), Tq, d->q_chunk, static_cast<const T*>(kpool), NB, d->bs, blk_len, pool_ids,
      nQB, q_bar, k_bar, status);
}

}  // namespace
}  // namespace pbsa

extern "C" int pbsa_score_blocks(const pbsa_dims* d, const void* q, int Tq, const void* kpool,
                                 int NB, const int32_t* blk_len, const int32_t* pool_ids,
                                 int n_pool, float* q_bar, float* k_bar, float* scores,
                                 float* mem_score, void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(Tq >= 1 && NB >= 1 && n_pool >= 0, PBSA_ERR_SHAPE,
                 "score_blocks: need Tq >= 1, NB >= 1, n_pool >= 0");
  PBSA_CHECK_ARG(q && kpool && blk_len && q_bar && k_bar && scores && mem_score, PBSA_ERR_ARG,
                 "score_blocks: NULL buffer");
  PBSA_CHECK_ARG(n_pool == 0 || pool_ids, PBSA_ERR_ARG, "score_blocks: pool_ids is NULL");
  PBSA_CHECK_ARG(aligned(q, 16) && aligned(kpool, 16), PBSA_ERR_ALIGN,
                 "score_blocks: q and kpool must be 16-byte aligned");
  PBSA_CHECK_ARG(aligned(q_bar, 4) && aligned(k_bar, 4) && aligned(scores, 4) &&
                     aligned(mem_score, 4) && aligned(blk_len, 4),
                 PBSA_ERR_ALIGN, "score_blocks: misaligned float/int buffer");
  const int nQB = qb_count(Tq, d->q_chunk, d->bs);
  PBSA_CHECK_ARG(static_cast<long>(d->B) * d->H <= 65535, PBSA_ERR_SHAPE,
                 "score_blocks: B*H must be <= 65535");
  int* status = device_status_ptr();
  PBSA_CHECK_ARG(status != nullptr, PBSA_ERR_CUDA, "score_blocks: no device status word");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d->dtype == PBSA_BF16) {
    if (d->D == 128)
      launch_pool<__nv_bfloat16, 128>(d, q, Tq, kpool, NB, blk_len, pool_ids, n_pool, nQB, q_bar,
                                      k_bar, status, s);
    else
      launch_pool<__nv_bfloat16, 64>(d, q, Tq, kpool, NB, blk_len, pool_ids, n_pool, nQB, q_bar,
                                     k_bar, status, s);
  } else {
    if (d->D == 128)
      launch_pool<float, 128>(d, q, Tq, kpool, NB, blk_len, pool_ids, n_pool, nQB, q_bar, k_bar,
                              status, s);
    else
      launch_pool<float, 64>(d, q, Tq, kpool, NB, blk_len, pool_ids, n_pool, nQB, q_bar, k_bar,
                             status, s);
  }
  PBSA_CHECK_LAUNCH("pool_kernel");
  dim3 grid((NB + kScoreJ - 1) / kScoreJ, d->B * d->H);
  const int qc = d->q_chunk > 0 ? d->q_chunk : Tq;
  const int per_group = (qc + d->bs - 1) / d->bs;
  const int groups = (Tq + qc - 1) / qc;
  if (d->D == 128)
    score_kernel<128><<<grid, 256, 0, s>>>(q_bar, k_bar, nQB, NB, d->scale, scores, mem_score,
                                           per_group, groups);
  else
    score_kernel<64><<<grid, 256, 0, s>>>(q_bar, k_bar, nQB, NB, d->scale, scores, mem_score,
                                          per_group, groups);
  PBSA_CHECK_LAUNCH("score_kernel");
  return PBSA_OK;
}
