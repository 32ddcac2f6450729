// a7: backward of the hybrid block-sparse attention on sm_100a tensor cores.
//
// The PBSA kernel serves training as well as inference (gist.science/es,
// section 3 "Contribuciones Clave", item "Kernel PBSA"; section 2
// "Entrenamiento": training runs with the dynamically updated cache).  The
// attended lists are constants of the backward pass.
//
// Launches:
//   prep   Delta_r = <dO_r, O_r> per query row, and a bitmap of the attended
//          (query block, key block) pairs;
//   rev    per (b,h): the reverse lists key block -> query blocks that attend
//          it, ascending (deterministic order of the dK/dV sums);
//   dkdv   one CTA per key block (128-row tile): for every query block i that
//          attends it, S^T = K Q_i^T and dP^T = V dO_i^T on tcgen05 into TMEM,
//          P^T = exp(S^T - LSE) and dS^T = P^T (dP^T - Delta) in fp32 by four
//          row warps, written to shared memory as bf16, then dV += P^T dO_i and
//          dK += dS^T Q_i accumulate in TMEM;
//   dq     one CTA per query tile: for every attended block j, S = Q K_j^T and
//          dP = dO V_j^T, dS = P (dP - Delta) written to TMEM as bf16, and
//          dQ += dS K_j in TMEM.
// Outputs are fp32; dK is scaled by `scale` at the end, dQ likewise.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "tc_sm100.cuh"
#include "tmap.h"

#include <mutex>
#include <string>

namespace pbsa {
namespace {

using namespace tc;

struct BwdParams {
  const int32_t* blk_len;
  const int32_t* blk_pos;
  const int32_t* idx;
  const int32_t* cnt;
  const __nv_bfloat16* o;
  const __nv_bfloat16* dO;
  const float* lse;
  float* delta;        // [BH, Tq]
  uint32_t* bitmap;    // [BH, NB, W32]
  int32_t* rev_off;    // [BH, NB + 1]
  int32_t* rev_q;      // [BH, nQB * Amax]
  float* dq;
  float* dk;
  float* dv;
  int B, H, Tq, q_chunk, q_pos0, NB, Amax, nQB, mask, W32, bs;
  float scale, scale_log2;
  int* status;
  int64_t limit_ns;
};

// ------------------------------------------------------------------ prep
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(BwdParams p) {
  pdl_wait();
  pdl_trigger();
  const int qi = blockIdx.x;
  const long bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int r0, n;
  qb_rows(qi, p.Tq, p.q_chunk, p.bs, r0, n);
  constexpr int PER = D / 32;  // bf16 per lane
  for (int r = warp; r < n; r += 8) {
    const long off = (bh * p.Tq + r0 + r) * D + lane * PER;
    float acc = 0.f;
    if (PER == 4) {
      const uint2 a = *reinterpret_cast<const uint2*>(p.o + off);
      const uint2 b = *reinterpret_cast<const uint2*>(p.dO + off);
      acc = bf16_lo(a.x) * bf16_lo(b.x) + bf16_hi(a.x) * bf16_hi(b.x) + bf16_lo(a.y) * bf16_lo(b.y) +
            bf16_hi(a.y) * bf16_hi(b.y);
    } else {
      const uint32_t a = *reinterpret_cast<const uint32_t*>(p.o + off);
      const uint32_t b = *reinterpret_cast<const uint32_t*>(p.dO + off);
      acc = bf16_lo(a) * bf16_lo(b) + bf16_hi(a) * bf16_hi(b);
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (lane == 0) p.delta[bh * p.Tq + r0 + r] = acc;
  }
  int c = p.cnt[bh * p.nQB + qi];
  c = max(0, min(c, p.Amax));
  const int32_t* ids = p.idx + (bh * p.nQB + qi) * p.Amax;
  for (int e = threadIdx.x; e < c; e += blockDim.x) {
    const int j = ids[e];
    if (j < 0 || j >= p.NB) {
      report_status(p.status, PBSA_ERR_ARG);
      continue;
    }
    atomicOr(&p.bitmap[(bh * p.NB + j) * p.W32 + (qi >> 5)], 1u << (qi & 31));
  }
}

// ------------------------------------------------------------------ reverse lists
__global__ void __launch_bounds__(256) bwd_rev_kernel(BwdParams p) {
  __shared__ int part[256];
  pdl_wait();
  pdl_trigger();
  const long bh = blockIdx.x;
  const int t = threadIdx.x;
  const int per = (p.NB + 255) / 256;
  const int j0 = t * per, j1 = min(p.NB, j0 + per);
  int mine = 0;
  for (int j = j0; j < j1; ++j)
    for (int w = 0; w < p.W32; ++w) mine += __popc(p.bitmap[(bh * p.NB + j) * p.W32 + w]);
  part[t] = mine;
  __syncthreads();
  // exclusive scan over 256 partial counts (Hillis-Steele in shared memory)
  for (int off = 1; off < 256; off <<= 1) {
    const int v = t >= off ? part[t - off] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  int pos = part[t] - mine;
  int32_t* roff = p.rev_off + bh * (p.NB + 1);
  int32_t* rq = p.rev_q + bh * static_cast<long>(p.nQB) * p.Amax;
  for (int j = j0; j < j1; ++j) {
    roff[j] = pos;
    for (int w = 0; w < p.W32; ++w) {
      uint32_t bits = p.bitmap[(bh * p.NB + j) * p.W32 + w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        rq[pos++] = w * 32 + b;
      }
    }
  }
  if (t == 255) roff[p.NB] = part[255];
}

// ------------------------------------------------------------------ dK / dV
// One CTA per key block j (the 128-row tiles K_j and V_j stay in shared
// memory), iterating over the query blocks i that attend it, in ascending
// order.  Q_i, dO_i and the rows' LSE and Delta stream through two stages.
// Tensor memory:
//   TM_ST   S^T = K_j Q_i^T (fp32).  The softmax warps overwrite its first 64
//           columns with P^T (bf16 pairs): the A operand of dV += P^T dO_i.
//   TM_DPT  dP^T = V_j dO_i^T.  Overwritten by dS^T = P^T (dP^T - Delta) (bf16
//           pairs): the A operand of dK += dS^T Q_i.
//   TM_DV, TM_DK  the accumulators.
// The MMA warp issues dV_i, S^T_{i+1}, dK_i, dP^T_{i+1} in that order: the
// tensor cores compute the next query block's S^T while the softmax warps
// form dS^T_i, and every reuse of a TMEM region is safe because tcgen05 MMAs
// issued by one thread run in order.  Eight softmax warps: warps w and w + 4
// own key rows 32(w % 4) .. +31 (their TMEM lanes) and take query columns
// [0, 64) and [64, 128) respectively, keeping their 64 probabilities in
// registers between the P^T and dS^T passes.  Each warp writes its bf16 pairs
// over columns it has already read: the pairs of query columns 16k .. 16k + 15
// (MMA k-step k) sit at TMEM column 64 (k / 4) + 8 (k % 4) of the region.
template <int D>
struct DkdvCfg {
  static constexpr int KB = D / 64;
  static constexpr int BOX = 128 * 128;            // 128 rows x 128 bytes
  static constexpr int TILE = KB * BOX;            // one 128-row operand tile
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;       // 2 stages
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;  // 2 stages
  static constexpr int OFF_LSE = OFF_DO + 2 * TILE;  // [2][128] floats (log2 units)
  static constexpr int OFF_DL = OFF_LSE + 2 * 128 * 4;
  static constexpr int OFF_BAR = OFF_DL + 2 * 128 * 4;
  static constexpr int B_KV = 0, B_QF = 1, B_QE = 3, B_SF = 5, B_DPF = 6, B_PF = 7, B_DSF = 8,
                       B_MMA = 9;
  static constexpr int NBAR = 10;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = 1024 + OFF_MISC + 16;
  static constexpr int TM_ST = 0, TM_DPT = 128, TM_DV = 256, TM_DK = 256 + D;
  static constexpr int TM_COLS = 512;
};

constexpr int kBwdThreads = 320;   // 8 softmax warps, producer, MMA issuer
constexpr int kBwdProducer = 8, kBwdMma = 9;

// TMEM column of the bf16 A operand for MMA k-step k (16 rows of K each)
__device__ __forceinline__ uint32_t a_col(int k) {
  return static_cast<uint32_t>((k >> 2) * 64 + (k & 3) * 8);
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                BwdParams p) {
  using C = DkdvCfg<D>;
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / p.NB;
  const int j = blockIdx.x - bh * p.NB;
  const int32_t* roff = p.rev_off + static_cast<long>(bh) * (p.NB + 1);
  const int32_t* rq = p.rev_q + static_cast<long>(bh) * p.nQB * p.Amax + roff[j];
  const int n = roff[j + 1] - roff[j];
  const int klen = min(max(p.blk_len[static_cast<long>(bh) * p.NB + j], 0), p.bs);
  const int kpos0 = p.blk_pos ? p.blk_pos[static_cast<long>(bh) * p.NB + j] : 0;

  const uint32_t sK = smem_u32(smem + C::OFF_K), sV = smem_u32(smem + C::OFF_V);
  const uint32_t sQ = smem_u32(smem + C::OFF_Q), sDO = smem_u32(smem + C::OFF_DO);
  float* s_lse = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* s_dl = reinterpret_cast<float*>(smem + C::OFF_DL);
  const uint32_t bar0 = smem_u32(smem + C::OFF_BAR);
  auto BAR = [&](int k) { return bar0 + 8u * static_cast<uint32_t>(k); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  if (tid == 0) {
    mbar_init(BAR(C::B_KV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(C::B_QF + s), 1);
      mbar_init(BAR(C::B_QE + s), 1);
    }
    mbar_init(BAR(C::B_SF), 1);
    mbar_init(BAR(C::B_DPF), 1);
    mbar_init(BAR(C::B_PF), 8);    // one arrival per softmax warp
    mbar_init(BAR(C::B_DSF), 8);
    mbar_init(BAR(C::B_MMA), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdProducer) {
    tmem_alloc(smem_u32(tmem_holder), C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == kBwdProducer) {
    // ---------------------------------------------------------- producer
    // K_j, V_j once; per query block: its LSE and Delta staged by the 32
    // lanes, then Q_i and dO_i by TMA into stage i & 1.
    if (n > 0) {
      int issued = 0;
      if (lane == 0) {
        const int kv_row = (bh * p.NB + j) * p.bs;
        mbar_expect_tx(BAR(C::B_KV), 2 * C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_2d(sK + kb * C::BOX, &tmK, BAR(C::B_KV), kb * 64, kv_row);
          tma_load_2d(sV + kb * C::BOX, &tmV, BAR(C::B_KV), kb * 64, kv_row);
        }
      }
      for (int it = 0; it < n; ++it) {
        const int s = it & 1;
        bool ok = true;
        if (it >= 2)
          ok = mbar_wait(BAR(C::B_QE + s), ((it >> 1) & 1) ^ 1, abort_flag, p.status, p.limit_ns);
        if (!__all_sync(0xffffffffu, ok)) break;
        int qrow0, qlen;
        qb_rows(rq[it], p.Tq, p.q_chunk, p.bs, qrow0, qlen);
        const long row_base = static_cast<long>(bh) * p.Tq + qrow0;
        for (int r = lane; r < 128; r += 32) {
          float l2 = INFINITY, dl = 0.f;
          if (r < qlen) {
            const float lse = p.lse[row_base + r];
            l2 = lse == -INFINITY ? INFINITY : lse * 1.4426950408889634f;
            dl = p.delta[row_base + r];
          }
          s_lse[s * 128 + r] = l2;
          s_dl[s * 128 + r] = dl;
        }
        __syncwarp();
        if (lane == 0) {
          mbar_expect_tx(BAR(C::B_QF + s), 2 * C::TILE);   // release: LSE/Delta staged
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb) {
            tma_load_2d(sQ + s * C::TILE + kb * C::BOX, &tmQ, BAR(C::B_QF + s), kb * 64,
                        static_cast<int>(row_base));
            tma_load_2d(sDO + s * C::TILE + kb * C::BOX, &tmDO, BAR(C::B_QF + s), kb * 64,
                        static_cast<int>(row_base));
          }
        }
        issued = it + 1;
      }
      if (lane == 0) {
        mbar_drain(BAR(C::B_KV), 0, p.status, p.limit_ns);
        for (int it = max(0, issued - 2); it < issued; ++it)
          mbar_drain(BAR(C::B_QF + (it & 1)), (it >> 1) & 1, p.status, p.limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == kBwdMma) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);  // K-major x K-major
      constexpr uint32_t id_kmn = idesc_bf16_f32(128, D, false, true);    // B MN-major
      auto issue_st = [&](int it) -> bool {   // S^T_it = K Q_it^T
        const int s = it & 1;
        if (!mbar_wait(BAR(C::B_QF + s), (it >> 1) & 1, abort_flag, p.status, p.limit_ns))
          return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * C::BOX + (k & 3) * 32;
          mma_ss(tmem + C::TM_ST, smem_desc_sw128(sK + off, 16, 1024),
                 smem_desc_sw128(sQ + s * C::TILE + off, 16, 1024), id_kk, k > 0);
        }
        mma_commit(BAR(C::B_SF));
        return true;
      };
      auto issue_dpt = [&](int it) {          // dP^T_it = V dO_it^T (Q/dO stage already full)
        const int s = it & 1;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * C::BOX + (k & 3) * 32;
          mma_ss(tmem + C::TM_DPT, smem_desc_sw128(sV + off, 16, 1024),
                 smem_desc_sw128(sDO + s * C::TILE + off, 16, 1024), id_kk, k > 0);
        }
        mma_commit(BAR(C::B_DPF));
      };
      bool ok = mbar_wait(BAR(C::B_KV), 0, abort_flag, p.status, p.limit_ns) && issue_st(0);
      if (ok) issue_dpt(0);
      for (int it = 0; ok && it < n; ++it) {
        const int s = it & 1;
        if (!mbar_wait(BAR(C::B_PF), it & 1, abort_flag, p.status, p.limit_ns)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 128 / 16; ++k)        // dV += P^T dO_it
          mma_ts(tmem + C::TM_DV, tmem + C::TM_ST + a_col(k),
                 smem_desc_sw128(sDO + s * C::TILE + k * 2048, C::BOX, 1024), id_kmn,
                 (it > 0 || k > 0) ? 1u : 0u);
        if (it + 1 < n && !issue_st(it + 1)) break;
        if (!mbar_wait(BAR(C::B_DSF), it & 1, abort_flag, p.status, p.limit_ns)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 128 / 16; ++k)        // dK += dS^T Q_it
          mma_ts(tmem + C::TM_DK, tmem + C::TM_DPT + a_col(k),
                 smem_desc_sw128(sQ + s * C::TILE + k * 2048, C::BOX, 1024), id_kmn,
                 (it > 0 || k > 0) ? 1u : 0u);
        mma_commit(BAR(C::B_QE + s));
        if (it + 1 < n) issue_dpt(it + 1);
      }
      mma_commit(BAR(C::B_MMA));
      mbar_drain(BAR(C::B_MMA), 0, p.status, p.limit_ns);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- softmax rows
    const int q4 = warp & 3, hh = warp >> 2;  // lane quarter, half of the query columns
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const int c = q4 * 32 + lane;           // key row of the tile
    const int col0 = hh * 64;               // this warp's query columns [col0, col0 + 64)
    const bool row_ok = c < klen;
    bool ok = true;
    const bool tok = p.mask == PBSA_MASK_TOKEN;
    int q_next = (tok && n > 0) ? rq[0] : 0;     // query block of the next step (token mask only)
    for (int it = 0; it < n; ++it) {
      const int s = it & 1;
      int qrow0 = 0;
      if (tok) {
        int qlen_unused;
        qb_rows(q_next, p.Tq, p.q_chunk, p.bs, qrow0, qlen_unused);
        if (it + 1 < n) q_next = rq[it + 1];
      }
      // stage s is full (LSE/Delta visible), then S^T_it is in TMEM
      ok = mbar_wait(BAR(C::B_QF + s), (it >> 1) & 1, abort_flag, p.status, p.limit_ns) &&
           mbar_wait(BAR(C::B_SF), it & 1, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float* lse_b = s_lse + s * 128;
      const float* dl_b = s_dl + s * 128;
      const int qpos0 = p.q_pos0 + qrow0;
      // first visible query column of this key row (rows past qlen have LSE = +inf)
      const int r_min = !row_ok ? 1 << 20 : (tok ? max(0, kpos0 + c - qpos0) : 0);
      float P[64];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t sv[32];
        tmem_ld32(tmem + lane_base + C::TM_ST + col0 + cc * 32, sv);
        // the 32 LSE values of this chunk: eight 128-bit broadcast reads
        float lv[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 t4 = reinterpret_cast<const float4*>(lse_b + col0 + cc * 32)[v];
          lv[4 * v] = t4.x; lv[4 * v + 1] = t4.y; lv[4 * v + 2] = t4.z; lv[4 * v + 3] = t4.w;
        }
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          // visible columns are r >= r_min; the exponent always runs (ex2(-inf) = 0)
          const int r = col0 + cc * 32 + e;
          const float x = __uint_as_float(sv[e]) * p.scale_log2 - lv[e];
          P[cc * 32 + e] = ex2(r >= r_min ? x : -INFINITY);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(P[cc * 32 + 2 * e], P[cc * 32 + 2 * e + 1]);
        // columns [col0 + 16cc, col0 + 16cc + 16) of S^T: this warp's, already read
        tmem_st16(tmem + lane_base + C::TM_ST + col0 + cc * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_PF));
      ok = mbar_wait(BAR(C::B_DPF), it & 1, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t dv[32];
        tmem_ld32(tmem + lane_base + C::TM_DPT + col0 + cc * 32, dv);
        float dlv[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 t4 = reinterpret_cast<const float4*>(dl_b + col0 + cc * 32)[v];
          dlv[4 * v] = t4.x; dlv[4 * v + 1] = t4.y; dlv[4 * v + 2] = t4.z; dlv[4 * v + 3] = t4.w;
        }
        tmem_wait_ld();
        uint32_t dk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int r = cc * 32 + 2 * e;
          const float d0 = P[r] * (__uint_as_float(dv[2 * e]) - dlv[2 * e]);
          const float d1 = P[r + 1] * (__uint_as_float(dv[2 * e + 1]) - dlv[2 * e + 1]);
          dk[e] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tmem + lane_base + C::TM_DPT + col0 + cc * 16, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_DSF));
    }
    // ---------------------------------------------------------- epilogue
    if (ok && n > 0) {
      ok = mbar_wait(BAR(C::B_MMA), 0, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const bool store = c < p.bs;
      float* dvrow = p.dv + ((static_cast<long>(bh) * p.NB + j) * p.bs + c) * D;
      float* dkrow = p.dk + ((static_cast<long>(bh) * p.NB + j) * p.bs + c) * D;
      // warps w and w + 4 store halves [0, D/2) and [D/2, D) of the row
#pragma unroll 1
      for (int cc = hh * (D / 64); cc < (hh + 1) * (D / 64); ++cc) {
        uint32_t a[32], b[32];
        if (n > 0) {
          tmem_ld32(tmem + lane_base + C::TM_DV + cc * 32, a);
          tmem_ld32(tmem + lane_base + C::TM_DK + cc * 32, b);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) { a[e] = 0u; b[e] = 0u; }
        }
        if (store) {
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            reinterpret_cast<float4*>(dvrow + cc * 32)[v] =
                make_float4(__uint_as_float(a[4 * v]), __uint_as_float(a[4 * v + 1]),
                            __uint_as_float(a[4 * v + 2]), __uint_as_float(a[4 * v + 3]));
            reinterpret_cast<float4*>(dkrow + cc * 32)[v] = make_float4(
                __uint_as_float(b[4 * v]) * p.scale, __uint_as_float(b[4 * v + 1]) * p.scale,
                __uint_as_float(b[4 * v + 2]) * p.scale, __uint_as_float(b[4 * v + 3]) * p.scale);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdProducer) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

// ------------------------------------------------------------------ dQ
// One CTA per query block (Q and dO stay in shared memory), iterating over its
// attended key blocks; K_j streams through NK stages and V_j through NV
// stages (K is needed until dQ_j, V only until dP_j).  Tensor memory:
//   TM_S0, TM_S1  S_j = Q K_j^T for alternate j; the softmax warps read S_j,
//                 keep P_j in registers and later overwrite S_j's first 64
//                 columns with dS_j = P_j (dP_j - Delta) (bf16 pairs): the A
//                 operand of dQ += dS_j K_j;
//   TM_DP         dP_j = dO V_j^T;
//   TM_DQ         the accumulator.
// The MMA warp issues dQ_j, dP_{j+1}, S_{j+2}: S_{j+1} is already computed
// when the softmax warps finish block j.
template <int D, int NK, int NV>
struct DqCfg {
  static constexpr int KB = D / 64;
  static constexpr int BOX = 128 * 128;
  static constexpr int TILE = KB * BOX;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + TILE;
  static constexpr int OFF_K = OFF_DO + TILE;
  static constexpr int OFF_V = OFF_K + NK * TILE;
  static constexpr int OFF_BAR = OFF_V + NV * TILE;
  static constexpr int B_Q = 0, B_KF = 1, B_KE = 1 + NK, B_VF = 1 + 2 * NK, B_VE = 1 + 2 * NK + NV,
                       B_SF = 1 + 2 * NK + 2 * NV, B_DPF = B_SF + 2, B_DSF = B_DPF + 1,
                       B_MMA = B_DSF + 1;
  static constexpr int NBAR = B_MMA + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = 1024 + OFF_MISC + 16;
  static constexpr int TM_S0 = 0, TM_DP = 128, TM_DQ = 256, TM_S1 = 256 + D;
  static constexpr int TM_COLS = 512;
};

template <int D, int NK, int NV>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
              const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              BwdParams p) {
  using C = DqCfg<D, NK, NV>;
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / p.nQB;
  const int qi = blockIdx.x - bh * p.nQB;
  int n = p.cnt[static_cast<long>(bh) * p.nQB + qi];
  n = max(0, min(n, p.Amax));
  int qrow0, qlen;
  qb_rows(qi, p.Tq, p.q_chunk, p.bs, qrow0, qlen);
  const int32_t* row_ids = p.idx + (static_cast<long>(bh) * p.nQB + qi) * p.Amax;

  const uint32_t sQ = smem_u32(smem + C::OFF_Q), sDO = smem_u32(smem + C::OFF_DO);
  const uint32_t sK = smem_u32(smem + C::OFF_K), sV = smem_u32(smem + C::OFF_V);
  const uint32_t bar0 = smem_u32(smem + C::OFF_BAR);
  auto BAR = [&](int k) { return bar0 + 8u * static_cast<uint32_t>(k); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  if (tid == 0) {
    mbar_init(BAR(C::B_Q), 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(BAR(C::B_KF + s), 1);
      mbar_init(BAR(C::B_KE + s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(BAR(C::B_VF + s), 1);
      mbar_init(BAR(C::B_VE + s), 1);
    }
    mbar_init(BAR(C::B_SF), 1);
    mbar_init(BAR(C::B_SF + 1), 1);
    mbar_init(BAR(C::B_DPF), 1);
    mbar_init(BAR(C::B_DSF), 8);    // one arrival per softmax warp
    mbar_init(BAR(C::B_MMA), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdProducer) {
    tmem_alloc(smem_u32(tmem_holder), C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // physical id of attended block jj (an invalid id is reported and read as
  // block 0, fully masked)
  auto block_id = [&](int jj) -> int {
    const int id = row_ids[jj];
    if (id < 0 || id >= p.NB) {
      report_status(p.status, PBSA_ERR_ARG);
      return -1;
    }
    return id;
  };

  if (warp == kBwdProducer) {
    // ---------------------------------------------------------- producer
    if (lane == 0 && n > 0) {
      const int q_row = bh * p.Tq + qrow0;
      mbar_expect_tx(BAR(C::B_Q), 2 * C::TILE);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb) {
        tma_load_2d(sQ + kb * C::BOX, &tmQ, BAR(C::B_Q), kb * 64, q_row);
        tma_load_2d(sDO + kb * C::BOX, &tmDO, BAR(C::B_Q), kb * 64, q_row);
      }
      int k_issued = 0, v_issued = 0;
      for (int jj = 0; jj < n; ++jj) {
        const int id = max(block_id(jj), 0);
        const int kv_row = (bh * p.NB + id) * p.bs;
        const int ks = jj % NK, vs = jj % NV;
        if (jj >= NK &&
            !mbar_wait(BAR(C::B_KE + ks), ((jj / NK) & 1) ^ 1, abort_flag, p.status, p.limit_ns))
          break;
        mbar_expect_tx(BAR(C::B_KF + ks), C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_2d(sK + ks * C::TILE + kb * C::BOX, &tmK, BAR(C::B_KF + ks), kb * 64, kv_row);
        k_issued = jj + 1;
        if (jj >= NV &&
            !mbar_wait(BAR(C::B_VE + vs), ((jj / NV) & 1) ^ 1, abort_flag, p.status, p.limit_ns))
          break;
        mbar_expect_tx(BAR(C::B_VF + vs), C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_2d(sV + vs * C::TILE + kb * C::BOX, &tmV, BAR(C::B_VF + vs), kb * 64, kv_row);
        v_issued = jj + 1;
      }
      mbar_drain(BAR(C::B_Q), 0, p.status, p.limit_ns);
      for (int jj = max(0, k_issued - NK); jj < k_issued; ++jj)
        mbar_drain(BAR(C::B_KF + jj % NK), (jj / NK) & 1, p.status, p.limit_ns);
      for (int jj = max(0, v_issued - NV); jj < v_issued; ++jj)
        mbar_drain(BAR(C::B_VF + jj % NV), (jj / NV) & 1, p.status, p.limit_ns);
    }
    __syncwarp();
  } else if (warp == kBwdMma) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_kmn = idesc_bf16_f32(128, D, false, true);
      auto issue_s = [&](int jj) -> bool {    // S_jj = Q K_jj^T
        const int ks = jj % NK;
        if (!mbar_wait(BAR(C::B_KF + ks), (jj / NK) & 1, abort_flag, p.status, p.limit_ns))
          return false;
        tc_fence_after();
        const uint32_t d_tm = tmem + ((jj & 1) ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * C::BOX + (k & 3) * 32;
          mma_ss(d_tm, smem_desc_sw128(sQ + off, 16, 1024),
                 smem_desc_sw128(sK + ks * C::TILE + off, 16, 1024), id_kk, k > 0);
        }
        mma_commit(BAR(C::B_SF + (jj & 1)));
        return true;
      };
      auto issue_dp = [&](int jj) -> bool {   // dP_jj = dO V_jj^T; frees V stage
        const int vs = jj % NV;
        if (!mbar_wait(BAR(C::B_VF + vs), (jj / NV) & 1, abort_flag, p.status, p.limit_ns))
          return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * C::BOX + (k & 3) * 32;
          mma_ss(tmem + C::TM_DP, smem_desc_sw128(sDO + off, 16, 1024),
                 smem_desc_sw128(sV + vs * C::TILE + off, 16, 1024), id_kk, k > 0);
        }
        mma_commit(BAR(C::B_DPF));
        mma_commit(BAR(C::B_VE + vs));
        return true;
      };
      bool ok = mbar_wait(BAR(C::B_Q), 0, abort_flag, p.status, p.limit_ns) && issue_s(0) &&
                issue_dp(0) && (n < 2 || issue_s(1));
      for (int jj = 0; ok && jj < n; ++jj) {
        if (!mbar_wait(BAR(C::B_DSF), jj & 1, abort_flag, p.status, p.limit_ns)) break;
        tc_fence_after();
        const int ks = jj % NK;
        const uint32_t ds_tm = tmem + ((jj & 1) ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int k = 0; k < 128 / 16; ++k)        // dQ += dS_jj K_jj
          mma_ts(tmem + C::TM_DQ, ds_tm + a_col(k),
                 smem_desc_sw128(sK + ks * C::TILE + k * 2048, C::BOX, 1024), id_kmn,
                 (jj > 0 || k > 0) ? 1u : 0u);
        mma_commit(BAR(C::B_KE + ks));
        // dP_{jj+1} overwrites dP_jj (read by the softmax before DSF_jj);
        // S_{jj+2} overwrites dS_jj (read by the dQ MMA just issued)
        if (jj + 1 < n && !issue_dp(jj + 1)) break;
        if (jj + 2 < n && !issue_s(jj + 2)) break;
      }
      mma_commit(BAR(C::B_MMA));
      mbar_drain(BAR(C::B_MMA), 0, p.status, p.limit_ns);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- softmax rows
    const int q4 = warp & 3, hh = warp >> 2;  // lane quarter, half of the key columns
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const int r = q4 * 32 + lane;           // query row of the tile
    const int col0 = hh * 64;               // this warp's key columns [col0, col0 + 64)
    const bool row_ok = r < qlen;
    float l2 = INFINITY, dl = 0.f;
    if (row_ok) {
      const float lse = p.lse[static_cast<long>(bh) * p.Tq + qrow0 + r];
      l2 = lse == -INFINITY ? INFINITY : lse * 1.4426950408889634f;
      dl = p.delta[static_cast<long>(bh) * p.Tq + qrow0 + r];
    }
    const int qpos = p.q_pos0 + qrow0 + r;
    // length and position of block jj, fetched one block ahead
    auto meta = [&](int jj, int& len, int& pos) {
      len = 0;
      pos = 0;
      if (jj < n) {
        const int id = block_id(jj);
        if (id >= 0) {
          len = min(max(p.blk_len[static_cast<long>(bh) * p.NB + id], 0), p.bs);
          pos = p.blk_pos ? p.blk_pos[static_cast<long>(bh) * p.NB + id] : 0;
        }
      }
    };
    int len_n, pos_n;
    meta(0, len_n, pos_n);
    bool ok = true;
    for (int jj = 0; jj < n; ++jj) {
      const int len = len_n, kpos0 = pos_n;
      meta(jj + 1, len_n, pos_n);
      ok = mbar_wait(BAR(C::B_SF + (jj & 1)), (jj >> 1) & 1, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_tm = tmem + lane_base + ((jj & 1) ? C::TM_S1 : C::TM_S0);
      int c_lim = row_ok ? len : 0;
      if (p.mask == PBSA_MASK_TOKEN) c_lim = min(c_lim, max(0, qpos - kpos0 + 1));
      float P[64];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t sv[32];
        tmem_ld32(s_tm + col0 + cc * 32, sv);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          // visible columns are col < c_lim; the exponent always runs (ex2(-inf) = 0)
          const int col = col0 + cc * 32 + e;
          const float x = __uint_as_float(sv[e]) * p.scale_log2 - l2;
          P[cc * 32 + e] = ex2(col < c_lim ? x : -INFINITY);
        }
      }
      ok = mbar_wait(BAR(C::B_DPF), jj & 1, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t dv[32];
        tmem_ld32(tmem + lane_base + C::TM_DP + col0 + cc * 32, dv);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int col = cc * 32 + 2 * e;
          pk[e] = pack_bf16x2(P[col] * (__uint_as_float(dv[2 * e]) - dl),
                              P[col + 1] * (__uint_as_float(dv[2 * e + 1]) - dl));
        }
        // columns [col0, col0 + 64) of S_jj are this warp's and were read above
        tmem_st16(s_tm + col0 + cc * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_DSF));
    }
    if (ok && n > 0) {
      ok = mbar_wait(BAR(C::B_MMA), 0, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      float* dqrow = p.dq + (static_cast<long>(bh) * p.Tq + qrow0 + r) * D;
      // warps w and w + 4 store halves [0, D/2) and [D/2, D) of the row
#pragma unroll 1
      for (int cc = hh * (D / 64); cc < (hh + 1) * (D / 64); ++cc) {
        uint32_t a[32];
        if (n > 0) {
          tmem_ld32(tmem + lane_base + C::TM_DQ + cc * 32, a);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) a[e] = 0u;
        }
        if (row_ok) {
#pragma unroll
          for (int v = 0; v < 8; ++v)
            reinterpret_cast<float4*>(dqrow + cc * 32)[v] = make_float4(
                __uint_as_float(a[4 * v]) * p.scale, __uint_as_float(a[4 * v + 1]) * p.scale,
                __uint_as_float(a[4 * v + 2]) * p.scale, __uint_as_float(a[4 * v + 3]) * p.scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdProducer) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}


struct BwdLayout {
  size_t delta, bitmap, rev_off, rev_q, total;
};

BwdLayout bwd_layout(const pbsa_dims* d, int Tq, int NB, int Amax) {
  const size_t BH = static_cast<size_t>(d->B) * d->H;
  const int nQB = qb_count(Tq, d->q_chunk, d->bs);
  const int W32 = (nQB + 31) / 32;
  BwdLayout L;
  size_t off = 0;
  L.delta = off; off = align_up(off + BH * Tq * 4, 256);
  L.bitmap = off; off = align_up(off + BH * NB * W32 * 4, 256);
  L.rev_off = off; off = align_up(off + BH * (NB + 1) * 4, 256);
  L.rev_q = off; off = align_up(off + BH * static_cast<size_t>(nQB) * Amax * 4, 256);
  L.total = off;
  return L;
}

// once per (kernel, device): the flag array is instantiated per kernel
template <auto Kern>
void opt_in_smem() {
  auto kern = Kern;
  static bool opted[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !opted[dev]) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (dev >= 0 && dev < 64) opted[dev] = true;
  }
}

template <int D>
int launch_bwd(const pbsa_dims* d, BwdParams& p, const CUtensorMap& mq, const CUtensorMap& mdo,
               const CUtensorMap& mk, const CUtensorMap& mv, void* ws, const BwdLayout& L,
               cudaStream_t s) {
  const int BH = d->B * d->H;
  if (cudaMemsetAsync(static_cast<char*>(ws) + L.bitmap, 0, L.rev_off - L.bitmap, s) !=
      cudaSuccess)
    PBSA_CHECK_LAUNCH("attn_bwd: memset");
  if (launch(bwd_prep_kernel<D>, dim3(p.nQB, BH), dim3(256), 0, s, p) != cudaSuccess)
    PBSA_CHECK_LAUNCH("bwd_prep_kernel");
  if (launch(bwd_rev_kernel, dim3(BH), dim3(256), 0, s, p) != cudaSuccess)
    PBSA_CHECK_LAUNCH("bwd_rev_kernel");
  {
    auto kern = bwd_dkdv_kernel<D>;
    opt_in_smem<bwd_dkdv_kernel<D>>();
    if (launch(kern, dim3(static_cast<unsigned>(BH) * p.NB), dim3(kBwdThreads), DkdvCfg<D>::SMEM, s, mq,
               mdo, mk, mv, p) != cudaSuccess)
      PBSA_CHECK_LAUNCH("bwd_dkdv_kernel");
  }
  {
    constexpr int NK = 3, NV = 2;
    auto kern = bwd_dq_kernel<D, NK, NV>;
    opt_in_smem<bwd_dq_kernel<D, NK, NV>>();
    const size_t smem = DqCfg<D, NK, NV>::SMEM;
    static_assert(DqCfg<128, 3, 2>::SMEM <= 227 * 1024, "dQ tiles exceed shared memory");
    if (launch(kern, dim3(static_cast<unsigned>(BH) * p.nQB), dim3(kBwdThreads), smem, s, mq, mdo, mk, mv,
               p) != cudaSuccess)
      PBSA_CHECK_LAUNCH("bwd_dq_kernel");
  }
  return PBSA_OK;
}

}  // namespace
}  // namespace pbsa

extern "C" size_t pbsa_attn_bwd_workspace(const pbsa_dims* d, int Tq, int NB, int Amax) {
  if (d == nullptr || Tq < 1 || NB < 1 || Amax < 1 || d->B < 1 || d->H < 1 || d->bs < 1) return 0;
  return pbsa::bwd_layout(d, Tq, NB, Amax).total;
}

extern "C" int pbsa_attn_bwd(const pbsa_dims* d, const void* q, int Tq, int q_pos0,
                             const void* kpool, const void* vpool, int NB,
                             const int32_t* blk_len, const int32_t* blk_pos, const int32_t* idx,
                             const int32_t* cnt, int Amax, int mask, const void* o,
                             const float* lse, const void* dO, float* dq, float* dk, float* dv,
                             void* workspace, size_t ws_bytes, void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(d->dtype == PBSA_BF16, PBSA_ERR_DTYPE, "attn_bwd: q/k/v must be bf16");
  PBSA_CHECK_ARG(q && kpool && vpool && blk_len && idx && cnt && o && lse && dO && dq && dk && dv,
                 PBSA_ERR_ARG, "attn_bwd: NULL buffer");
  PBSA_CHECK_ARG(mask == PBSA_MASK_CHUNK || (mask == PBSA_MASK_TOKEN && blk_pos), PBSA_ERR_ARG,
                 "attn_bwd: bad mask, or token mask without blk_pos");
  PBSA_CHECK_ARG(Tq >= 1 && NB >= 1 && Amax >= 1, PBSA_ERR_SHAPE,
                 "attn_bwd: need Tq >= 1, NB >= 1, Amax >= 1");
  PBSA_CHECK_ARG(aligned(q, 16) && aligned(kpool, 16) && aligned(vpool, 16) && aligned(o, 16) &&
                     aligned(dO, 16) && aligned(dq, 16) && aligned(dk, 16) && aligned(dv, 16),
                 PBSA_ERR_ALIGN, "attn_bwd: tensors must be 16-byte aligned");
  const long BH = static_cast<long>(d->B) * d->H;
  const int nQB = qb_count(Tq, d->q_chunk, d->bs);
  PBSA_CHECK_ARG(BH * Tq < (1L << 31) && BH * NB * d->bs < (1L << 31), PBSA_ERR_SHAPE,
                 "attn_bwd: tensor rows must be < 2^31");
  PBSA_CHECK_ARG(BH * NB < (1L << 31) && BH <= 65535 && nQB <= 65535, PBSA_ERR_SHAPE,
                 "attn_bwd: grid too large");
  const BwdLayout L = bwd_layout(d, Tq, NB, Amax);
  PBSA_CHECK_ARG(workspace && ws_bytes >= L.total && aligned(workspace, 256), PBSA_ERR_WORKSPACE,
                 "attn_bwd: workspace missing, too small or not 256-byte aligned (need " +
                     std::to_string(L.total) + " bytes)");
  int* status = device_status_ptr();
  PBSA_CHECK_ARG(status != nullptr, PBSA_ERR_CUDA, "attn_bwd: no device status word");
  CUtensorMap mq, mdo, mk, mv;
  if ((rc = make_tmap_bf16_2d(&mq, q, BH * Tq, d->D, 128, 64))) return rc;
  if ((rc = make_tmap_bf16_2d(&mdo, dO, BH * Tq, d->D, 128, 64))) return rc;
  if ((rc = make_tmap_bf16_2d(&mk, kpool, BH * NB * d->bs, d->D, 128, 64))) return rc;
  if ((rc = make_tmap_bf16_2d(&mv, vpool, BH * NB * d->bs, d->D, 128, 64))) return rc;
  char* ws = static_cast<char*>(workspace);
  BwdParams p;
  p.blk_len = blk_len; p.blk_pos = blk_pos; p.idx = idx; p.cnt = cnt;
  p.o = static_cast<const __nv_bfloat16*>(o);
  p.dO = static_cast<const __nv_bfloat16*>(dO);
  p.lse = lse;
  p.delta = reinterpret_cast<float*>(ws + L.delta);
  p.bitmap = reinterpret_cast<uint32_t*>(ws + L.bitmap);
  p.rev_off = reinterpret_cast<int32_t*>(ws + L.rev_off);
  p.rev_q = reinterpret_cast<int32_t*>(ws + L.rev_q);
  p.dq = dq; p.dk = dk; p.dv = dv;
  p.B = d->B; p.H = d->H; p.Tq = Tq; p.q_chunk = d->q_chunk; p.q_pos0 = q_pos0; p.NB = NB; p.Amax = Amax; p.nQB = nQB;
  p.mask = mask; p.W32 = (nQB + 31) / 32; p.bs = d->bs;
  p.scale = d->scale; p.scale_log2 = d->scale * 1.4426950408889634f;
  p.status = status; p.limit_ns = wait_limit_ns();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d->D == 128) return launch_bwd<128>(d, p, mq, mdo, mk, mv, workspace, L, s);
  return launch_bwd<64>(d, p, mq, mdo, mk, mv, workspace, L, s);
}

// ---------------------------------------------------------------------------
// Backward without a caller-provided workspace.
//
// Some callers cannot hand this library a device buffer: a host process that
// owns all device memory through its own pool and gives plugins no allocator
// hook, or latency-critical code that must never enter the CUDA allocator
// (cudaMalloc can synchronise the device and take milliseconds).  For them the
// scratch of the backward (Delta, the attended-pair bitmap and the reverse
// lists) lives in a fixed array of device memory that is part of the library
// image: every GPU that loads libpbsa.so holds these 16 MiB until the process
// exits.
// ---------------------------------------------------------------------------
namespace pbsa {
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(16) << 20;
__device__ __align__(256) unsigned char g_bwd_scratch[kNoAllocScratchBytes];

// Device address of g_bwd_scratch on the current device.  In host code the
// array's name only stands in for the device symbol, so the address is looked
// up once per device (with that device current) and cached.
void* noalloc_scratch(std::string* err) {
  static void* ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    *err = std::string("cannot query the current device: ") + cudaGetErrorString(e);
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_bwd_scratch);
    if (e != cudaSuccess || p == nullptr) {
      *err = std::string("cudaGetSymbolAddress of the backward scratch failed: ") +
             cudaGetErrorString(e);
      return nullptr;
    }
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

}  // namespace
}  // namespace pbsa

extern "C" size_t pbsa_attn_bwd_noalloc_max_scratch(void) { return pbsa::kNoAllocScratchBytes; }

extern "C" int pbsa_attn_bwd_noalloc(const pbsa_dims* d, const void* q, int Tq, int q_pos0,
                                     const void* kpool, const void* vpool, int NB,
                                     const int32_t* blk_len, const int32_t* blk_pos,
                                     const int32_t* idx, const int32_t* cnt, int Amax, int mask,
                                     const void* o, const float* lse, const void* dO, float* dq,
                                     float* dk, float* dv, void* stream) {
  using namespace pbsa;
  int rc = common_dims_check(d);
  if (rc) return rc;
  PBSA_CHECK_ARG(Tq >= 1 && NB >= 1 && Amax >= 1, PBSA_ERR_SHAPE,
                 "attn_bwd_noalloc: need Tq >= 1, NB >= 1, Amax >= 1");
  const size_t need = pbsa_attn_bwd_workspace(d, Tq, NB, Amax);
  PBSA_CHECK_ARG(need > 0 && need <= kNoAllocScratchBytes, PBSA_ERR_WORKSPACE,
                 "attn_bwd_noalloc: this problem needs " + std::to_string(need) +
                     " bytes of scratch, more than the built-in " +
                     std::to_string(kNoAllocScratchBytes) +
                     " bytes; use pbsa_attn_bwd with a workspace");
  std::string err;
  void* ws = noalloc_scratch(&err);
  PBSA_CHECK_ARG(ws != nullptr, PBSA_ERR_CUDA, "attn_bwd_noalloc: " + err);
  // The shared scratch keeps the previous call's contents; the backward clears
  // the part that must start at zero (the pair bitmap) and fully rewrites the rest.
  return pbsa_attn_bwd(d, q, Tq, q_pos0, kpool, vpool, NB, blk_len, blk_pos, idx, cnt, Amax, mask,
                       o, lse, dO, dq, dk, dv, ws, kNoAllocScratchBytes, stream);
}
