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

// ------------------------------------------------------------------ shared
// Write 8 consecutive bf16 (columns 8q..8q+7 of row `row`) of a 128-row,
// K-major, 128-byte-swizzled operand tile made of 64-column atoms.
__device__ __forceinline__ void st_sw128_chunk(uint8_t* tile, int row, int col8, uint4 v) {
  const int atom = col8 >> 3;          // 8 chunks of 8 columns per atom
  const int q = col8 & 7;
  uint8_t* dst = tile + atom * (128 * 128) + row * 128 + ((q ^ (row & 7)) << 4);
  *reinterpret_cast<uint4*>(dst) = v;
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ dK / dV
template <int D>
struct DkdvCfg {
  static constexpr int KB = D / 64;
  static constexpr int BOX = 128 * 128;            // 128 rows x 128 bytes
  static constexpr int TILE = KB * BOX;            // one 128-row operand tile
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;
  static constexpr int OFF_DO = OFF_Q + TILE;
  static constexpr int OFF_PT = OFF_DO + TILE;     // P^T, 128 x 128 bf16
  static constexpr int OFF_DST = OFF_PT + 2 * BOX; // dS^T
  static constexpr int OFF_LSE = OFF_DST + 2 * BOX;  // [2][128] floats
  static constexpr int OFF_DL = OFF_LSE + 2 * 128 * 4;
  static constexpr int OFF_BAR = OFF_DL + 2 * 128 * 4;
  // barriers
  static constexpr int B_KV = 0, B_QF = 1, B_QE = 2, B_SF = 3, B_PF = 4, B_DSF = 5, B_MMA = 6;
  static constexpr int B_ST = 7;   // + parity (2): LSE/Delta staged by all 128 row threads
  static constexpr int NBAR = 9;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = 1024 + OFF_MISC + 16;
  static constexpr int TM_ST = 0, TM_DPT = 128, TM_DV = 256, TM_DK = 256 + D;
  static constexpr int TM_COLS = 512;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
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
  const uint32_t sPT = smem_u32(smem + C::OFF_PT), sDST = smem_u32(smem + C::OFF_DST);
  float* s_lse = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* s_dl = reinterpret_cast<float*>(smem + C::OFF_DL);
  const uint32_t bar0 = smem_u32(smem + C::OFF_BAR);
  auto BAR = [&](int k) { return bar0 + 8u * static_cast<uint32_t>(k); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  if (tid == 0) {
    mbar_init(BAR(C::B_KV), 1);
    mbar_init(BAR(C::B_QF), 1);
    mbar_init(BAR(C::B_QE), 1);
    mbar_init(BAR(C::B_SF), 1);
    mbar_init(BAR(C::B_PF), 128);
    mbar_init(BAR(C::B_DSF), 128);
    mbar_init(BAR(C::B_MMA), 1);
    mbar_init(BAR(C::B_ST), 128);
    mbar_init(BAR(C::B_ST + 1), 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_holder), C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 4) {
    if (lane == 0 && n > 0) {
      const int kv_row = (bh * p.NB + j) * p.bs;
      mbar_expect_tx(BAR(C::B_KV), 2 * C::TILE);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb) {
        tma_load_2d(sK + kb * C::BOX, &tmK, BAR(C::B_KV), kb * 64, kv_row);
        tma_load_2d(sV + kb * C::BOX, &tmV, BAR(C::B_KV), kb * 64, kv_row);
      }
      int issued = 0;
      for (int it = 0; it < n; ++it) {
        if (it > 0 && !mbar_wait(BAR(C::B_QE), (it - 1) & 1, abort_flag, p.status, p.limit_ns))
          break;
        int qrow0, qlen;
        qb_rows(rq[it], p.Tq, p.q_chunk, p.bs, qrow0, qlen);
        const int q_row = bh * p.Tq + qrow0;
        mbar_expect_tx(BAR(C::B_QF), 2 * C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_2d(sQ + kb * C::BOX, &tmQ, BAR(C::B_QF), kb * 64, q_row);
          tma_load_2d(sDO + kb * C::BOX, &tmDO, BAR(C::B_QF), kb * 64, q_row);
        }
        issued = it + 1;
      }
      mbar_drain(BAR(C::B_KV), 0, p.status, p.limit_ns);
      if (issued > 0) mbar_drain(BAR(C::B_QF), (issued - 1) & 1, p.status, p.limit_ns);
    }
    __syncwarp();
  } else if (warp == 5) {
    if (lane == 0 && n > 0) {
      constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);  // K-major x K-major
      constexpr uint32_t id_kmn = idesc_bf16_f32(128, D, false, true);    // B MN-major
      if (mbar_wait(BAR(C::B_KV), 0, abort_flag, p.status, p.limit_ns)) {
        for (int it = 0; it < n; ++it) {
          if (!mbar_wait(BAR(C::B_QF), it & 1, abort_flag, p.status, p.limit_ns)) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * C::BOX + (k & 3) * 32;
            mma_ss(tmem + C::TM_ST, smem_desc_sw128(sK + off, 16, 1024),
                   smem_desc_sw128(sQ + off, 16, 1024), id_kk, k > 0);
            mma_ss(tmem + C::TM_DPT, smem_desc_sw128(sV + off, 16, 1024),
                   smem_desc_sw128(sDO + off, 16, 1024), id_kk, k > 0);
          }
          mma_commit(BAR(C::B_SF));
          if (!mbar_wait(BAR(C::B_PF), it & 1, abort_flag, p.status, p.limit_ns)) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 128 / 16; ++k) {
            const uint32_t aoff = (k >> 2) * C::BOX + (k & 3) * 32;
            mma_ss(tmem + C::TM_DV, smem_desc_sw128(sPT + aoff, 16, 1024),
                   smem_desc_sw128(sDO + k * 2048, C::BOX, 1024), id_kmn, (it > 0 || k > 0));
          }
          if (!mbar_wait(BAR(C::B_DSF), it & 1, abort_flag, p.status, p.limit_ns)) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 128 / 16; ++k) {
            const uint32_t aoff = (k >> 2) * C::BOX + (k & 3) * 32;
            mma_ss(tmem + C::TM_DK, smem_desc_sw128(sDST + aoff, 16, 1024),
                   smem_desc_sw128(sQ + k * 2048, C::BOX, 1024), id_kmn, (it > 0 || k > 0));
          }
          mma_commit(BAR(C::B_QE));
        }
      }
      mma_commit(BAR(C::B_MMA));
      mbar_drain(BAR(C::B_MMA), 0, p.status, p.limit_ns);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- row warps
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int c = tid;                      // key row in the tile
    bool ok = true;
    for (int it = 0; it < n; ++it) {
      const int qi = rq[it];
      int qrow0, qlen;
      qb_rows(qi, p.Tq, p.q_chunk, p.bs, qrow0, qlen);
      float* lse_b = s_lse + (it & 1) * 128;
      float* dl_b = s_dl + (it & 1) * 128;
      {
        const int r = tid;
        float l2 = INFINITY, dl = 0.f;
        if (r < qlen) {
          const float lse = p.lse[static_cast<long>(bh) * p.Tq + qrow0 + r];
          l2 = lse == -INFINITY ? INFINITY : lse * 1.4426950408889634f;
          dl = p.delta[static_cast<long>(bh) * p.Tq + qrow0 + r];
        }
        lse_b[r] = l2;
        dl_b[r] = dl;
      }
      // every row thread needs all 128 staged values: bounded handshake
      mbar_arrive(BAR(C::B_ST + (it & 1)));
      ok = mbar_wait(BAR(C::B_ST + (it & 1)), (it >> 1) & 1, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ok = mbar_wait(BAR(C::B_SF), it & 1, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int qpos0 = p.q_pos0 + qrow0;
      const bool row_ok = c < klen;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sv[32], dv[32];
        tmem_ld32(tmem + lane_base + C::TM_ST + cc * 32, sv);
        tmem_ld32(tmem + lane_base + C::TM_DPT + cc * 32, dv);
        tmem_wait_ld();
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float pv[2], ds[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int r = cc * 32 + e + u;
            bool vis = row_ok && r < p.bs;
            if (p.mask == PBSA_MASK_TOKEN) vis = vis && (kpos0 + c <= qpos0 + r);
            const float x = __uint_as_float(sv[e + u]) * p.scale_log2 - lse_b[r];
            pv[u] = vis ? ex2(x) : 0.f;
            ds[u] = pv[u] * (__uint_as_float(dv[e + u]) - dl_b[r]);
          }
          pk[e >> 1] = pack_bf16x2(pv[0], pv[1]);
          dk[e >> 1] = pack_bf16x2(ds[0], ds[1]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          st_sw128_chunk(smem + C::OFF_PT, c, cc * 4 + q,
                         make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]));
          st_sw128_chunk(smem + C::OFF_DST, c, cc * 4 + q,
                         make_uint4(dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]));
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(BAR(C::B_PF));
      mbar_arrive(BAR(C::B_DSF));
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
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
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
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

// ------------------------------------------------------------------ dQ
template <int D, int NST>
struct DqCfg {
  static constexpr int KB = D / 64;
  static constexpr int BOX = 128 * 128;
  static constexpr int TILE = KB * BOX;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + TILE;
  static constexpr int OFF_K = OFF_DO + TILE;
  static constexpr int OFF_V = OFF_K + NST * TILE;
  static constexpr int OFF_BAR = OFF_V + NST * TILE;
  static constexpr int B_Q = 0, B_KF = 1, B_VF = 1 + NST, B_KVE = 1 + 2 * NST;
  static constexpr int B_SF = 1 + 3 * NST, B_DSF = 2 + 3 * NST, B_MMA = 3 + 3 * NST;
  static constexpr int NBAR = 4 + 3 * NST;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_IDS = OFF_MISC + 16;
  static constexpr int TM_S = 0, TM_DP = 128, TM_DQ = 256, TM_DS = 256 + D;
  static constexpr int TM_COLS = 512;
  static size_t smem_bytes(int Amax) { return 1024 + OFF_IDS + 3 * 4 * static_cast<size_t>(Amax); }
};

template <int D, int NST>
__global__ void __launch_bounds__(192, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
              const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              BwdParams p) {
  using C = DqCfg<D, NST>;
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

  const uint32_t sQ = smem_u32(smem + C::OFF_Q), sDO = smem_u32(smem + C::OFF_DO);
  const uint32_t sK = smem_u32(smem + C::OFF_K), sV = smem_u32(smem + C::OFF_V);
  const uint32_t bar0 = smem_u32(smem + C::OFF_BAR);
  auto BAR = [&](int k) { return bar0 + 8u * static_cast<uint32_t>(k); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* s_ids = reinterpret_cast<int*>(smem + C::OFF_IDS);
  int* s_len = s_ids + p.Amax;
  int* s_pos = s_len + p.Amax;

  if (tid == 0) {
    mbar_init(BAR(C::B_Q), 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(BAR(C::B_KF + s), 1);
      mbar_init(BAR(C::B_VF + s), 1);
      mbar_init(BAR(C::B_KVE + s), 1);
    }
    mbar_init(BAR(C::B_SF), 1);
    mbar_init(BAR(C::B_DSF), 128);
    mbar_init(BAR(C::B_MMA), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const int32_t* row_ids = p.idx + (static_cast<long>(bh) * p.nQB + qi) * p.Amax;
  for (int e = tid; e < n; e += blockDim.x) {
    int id = row_ids[e];
    int len = 0, pos = 0;
    if (id < 0 || id >= p.NB) {
      report_status(p.status, PBSA_ERR_ARG);
      id = 0;
    } else {
      len = min(max(p.blk_len[static_cast<long>(bh) * p.NB + id], 0), p.bs);
      pos = p.blk_pos ? p.blk_pos[static_cast<long>(bh) * p.NB + id] : 0;
    }
    s_ids[e] = id;
    s_len[e] = len;
    s_pos[e] = pos;
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_holder), C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 4) {
    if (lane == 0 && n > 0) {
      const int q_row = bh * p.Tq + qrow0;
      mbar_expect_tx(BAR(C::B_Q), 2 * C::TILE);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb) {
        tma_load_2d(sQ + kb * C::BOX, &tmQ, BAR(C::B_Q), kb * 64, q_row);
        tma_load_2d(sDO + kb * C::BOX, &tmDO, BAR(C::B_Q), kb * 64, q_row);
      }
      int issued = 0;
      for (int jj = 0; jj < n; ++jj) {
        const int s = jj % NST;
        if (jj >= NST &&
            !mbar_wait(BAR(C::B_KVE + s), ((jj / NST) & 1) ^ 1, abort_flag, p.status, p.limit_ns))
          break;
        const int kv_row = (bh * p.NB + s_ids[jj]) * p.bs;
        mbar_expect_tx(BAR(C::B_KF + s), C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_2d(sK + s * C::TILE + kb * C::BOX, &tmK, BAR(C::B_KF + s), kb * 64, kv_row);
        mbar_expect_tx(BAR(C::B_VF + s), C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_2d(sV + s * C::TILE + kb * C::BOX, &tmV, BAR(C::B_VF + s), kb * 64, kv_row);
        issued = jj + 1;
      }
      mbar_drain(BAR(C::B_Q), 0, p.status, p.limit_ns);
      for (int s = 0; s < NST && s < issued; ++s) {
        const int jl = s + ((issued - 1 - s) / NST) * NST;
        mbar_drain(BAR(C::B_KF + s), (jl / NST) & 1, p.status, p.limit_ns);
        mbar_drain(BAR(C::B_VF + s), (jl / NST) & 1, p.status, p.limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    if (lane == 0 && n > 0) {
      constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_kmn = idesc_bf16_f32(128, D, false, true);
      if (mbar_wait(BAR(C::B_Q), 0, abort_flag, p.status, p.limit_ns)) {
        for (int jj = 0; jj < n; ++jj) {
          const int s = jj % NST;
          if (!mbar_wait(BAR(C::B_KF + s), (jj / NST) & 1, abort_flag, p.status, p.limit_ns)) break;
          if (!mbar_wait(BAR(C::B_VF + s), (jj / NST) & 1, abort_flag, p.status, p.limit_ns)) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * C::BOX + (k & 3) * 32;
            mma_ss(tmem + C::TM_S, smem_desc_sw128(sQ + off, 16, 1024),
                   smem_desc_sw128(sK + s * C::TILE + off, 16, 1024), id_kk, k > 0);
            mma_ss(tmem + C::TM_DP, smem_desc_sw128(sDO + off, 16, 1024),
                   smem_desc_sw128(sV + s * C::TILE + off, 16, 1024), id_kk, k > 0);
          }
          mma_commit(BAR(C::B_SF));
          if (!mbar_wait(BAR(C::B_DSF), jj & 1, abort_flag, p.status, p.limit_ns)) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 128 / 16; ++k)
            mma_ts(tmem + C::TM_DQ, tmem + C::TM_DS + k * 8,
                   smem_desc_sw128(sK + s * C::TILE + k * 2048, C::BOX, 1024), id_kmn,
                   (jj > 0 || k > 0));
          mma_commit(BAR(C::B_KVE + s));
        }
      }
      mma_commit(BAR(C::B_MMA));
      mbar_drain(BAR(C::B_MMA), 0, p.status, p.limit_ns);
    }
    __syncwarp();
  } else {
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int r = tid;
    const bool row_ok = r < qlen;
    float l2 = INFINITY, dl = 0.f;
    if (row_ok) {
      const float lse = p.lse[static_cast<long>(bh) * p.Tq + qrow0 + r];
      l2 = lse == -INFINITY ? INFINITY : lse * 1.4426950408889634f;
      dl = p.delta[static_cast<long>(bh) * p.Tq + qrow0 + r];
    }
    const int qpos = p.q_pos0 + qrow0 + r;
    bool ok = true;
    for (int jj = 0; jj < n; ++jj) {
      ok = mbar_wait(BAR(C::B_SF), jj & 1, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int len = s_len[jj];
      const int kpos0 = s_pos[jj];
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sv[32], dv[32];
        tmem_ld32(tmem + lane_base + C::TM_S + cc * 32, sv);
        tmem_ld32(tmem + lane_base + C::TM_DP + cc * 32, dv);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float ds[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int col = cc * 32 + e + u;
            bool vis = row_ok && col < len;
            if (p.mask == PBSA_MASK_TOKEN) vis = vis && (kpos0 + col <= qpos);
            const float pv = vis ? ex2(__uint_as_float(sv[e + u]) * p.scale_log2 - l2) : 0.f;
            ds[u] = pv * (__uint_as_float(dv[e + u]) - dl);
          }
          pk[e >> 1] = pack_bf16x2(ds[0], ds[1]);
        }
        tmem_st16(tmem + lane_base + C::TM_DS + cc * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(C::B_DSF));
    }
    if (ok && n > 0) {
      ok = mbar_wait(BAR(C::B_MMA), 0, abort_flag, p.status, p.limit_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      float* dqrow = p.dq + (static_cast<long>(bh) * p.Tq + qrow0 + r) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
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
  if (warp == 4) {
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
    if (launch(kern, dim3(static_cast<unsigned>(BH) * p.NB), dim3(192), DkdvCfg<D>::SMEM, s, mq,
               mdo, mk, mv, p) != cudaSuccess)
      PBSA_CHECK_LAUNCH("bwd_dkdv_kernel");
  }
  {
    constexpr int NST = 2;
    auto kern = bwd_dq_kernel<D, NST>;
    opt_in_smem<bwd_dq_kernel<D, NST>>();
    const size_t smem = DqCfg<D, NST>::smem_bytes(p.Amax);
    PBSA_CHECK_ARG(smem <= 227 * 1024, PBSA_ERR_SHAPE, "attn_bwd: Amax too large");
    if (launch(kern, dim3(static_cast<unsigned>(BH) * p.nQB), dim3(192), smem, s, mq, mdo, mk, mv,
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
