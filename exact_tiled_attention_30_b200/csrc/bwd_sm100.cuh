// Backward kernels of exact tiled attention for sm_100a (B200).
//
// The pages benchmark the backward pass (reproduction page of the
// FlashAttention-2 paper, Figure 6a-d) but print no equations; the kernels
// compute the chain-rule gradients of softmax attention, recomputing P from the
// saved row log-sum-exp instead of storing it (the N x N matrices stay on chip,
// as in the forward pass: "FlashAttention (v2)" glossary page, definition):
//   D_i   = sum_c dO_ic O_ic                               (preprocess)
//   P_ij  = exp(scale * q_i.k_j - LSE_i),  dP_ij = dO_i.v_j
//   dS_ij = P_ij (dP_ij - D_i)
//   dV_j  = sum_i P_ij dO_i,  dK_j = scale sum_i dS_ij q_i,  dQ_i = scale sum_j dS_ij k_j
//
// Kernels, all on the caller's stream:
//   1. fa2_bwd_pre: D and LSE * log2(e) into the workspace (rows padded to a
//      multiple of 128: D = 0, LSE = +inf there so P vanishes), dQ accumulator
//      zeroed. HBM-bound.
//   2. fa2_bwd_kernel: one CTA per (128-key block, batch*head), parallel over key
//      blocks. K_j, V_j stay in shared memory; query blocks i stream through a
//      TMA ring (causal: only i >= j). Per block: S^T = K Q_i^T and dP^T = V dO_i^T
//      into tensor memory (keys on TMEM lanes), four warps (one key row per
//      thread) form P^T and dS^T in bf16 into swizzled shared memory; then
//      dV += P^T dO_i, dK += dS^T Q_i (accumulated in TMEM across all i) and
//      dQ_i = dS K_j (the same dS^T buffer read MN-major), which the four warps
//      add into the fp32 accumulator with vector reductions.
//   3. fa2_bwd_dq_convert: dQ = bf16(scale * accumulator).
#pragma once

#include "sm100_ptx.cuh"

namespace fa2 {

// ------------------------------------------------------------- preprocess (B1)
struct BwdPreParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;
  float* dq_acc;   // [BH][Np][d]
  float* delta;    // [BH][Np]
  float* lse2;     // [BH][Np]
  int N;
  int Np;
  long long rows;  // BH * Np
};

// 16 threads per row (d = 128) or 8 (d = 64), 16 bytes of O and dO per thread.
template <int D>
__global__ void __launch_bounds__(256) fa2_bwd_pre_kernel(const BwdPreParams p) {
  constexpr int TPR = D / 8;            // threads per row
  constexpr int RPB = 256 / TPR;        // rows per block per sweep
  const int sub = threadIdx.x % TPR;
  const long long stride = static_cast<long long>(gridDim.x) * RPB;
  for (long long r = static_cast<long long>(blockIdx.x) * RPB + threadIdx.x / TPR; r < p.rows;
       r += stride) {
    const long long bh = r / p.Np;
    const int n = static_cast<int>(r - bh * p.Np);
    float acc = 0.f;
    if (n < p.N) {
      const size_t off = (static_cast<size_t>(bh) * p.N + n) * D + sub * 8;
      const uint4 ov = *reinterpret_cast<const uint4*>(p.o + off);
      const uint4 dv = *reinterpret_cast<const uint4*>(p.dout + off);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
      const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 a = __bfloat1622float2(o2[i]);
        const float2 b = __bfloat1622float2(d2[i]);
        acc = fmaf(a.x, b.x, acc);
        acc = fmaf(a.y, b.y, acc);
      }
    }
#pragma unroll
    for (int w = TPR / 2; w > 0; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w, TPR);
    float4* z = reinterpret_cast<float4*>(p.dq_acc + static_cast<size_t>(r) * D + sub * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (sub == 0) {
      p.delta[r] = acc;
      p.lse2[r] = (n < p.N) ? p.lse[static_cast<size_t>(bh) * p.N + n] * 1.4426950408889634f
                            : INFINITY;
    }
  }
}

// ---------------------------------------------------------- dQ convert (B3a)
struct BwdConvertParams {
  const float* dq_acc;  // [BH][Np][d]
  __nv_bfloat16* dq;    // [BH][N][d]
  int N;
  int Np;
  int d;
  long long total8;     // BH * N * d / 8
  float scale;
};

__global__ void __launch_bounds__(256) fa2_bwd_dq_convert_kernel(const BwdConvertParams p) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const int per_row8 = p.d / 8;
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < p.total8;
       t += stride) {
    const long long row = t / per_row8;  // bh * N + n
    const int c8 = static_cast<int>(t - row * per_row8);
    const long long bh = row / p.N;
    const long long n = row - bh * p.N;
    const float4* src =
        reinterpret_cast<const float4*>(p.dq_acc + (static_cast<size_t>(bh) * p.Np + n) * p.d + c8 * 8);
    const float4 a = src[0];
    const float4 b = src[1];
    uint4 w;
    w.x = pack_bf16(a.x * p.scale, a.y * p.scale);
    w.y = pack_bf16(a.z * p.scale, a.w * p.scale);
    w.z = pack_bf16(b.x * p.scale, b.y * p.scale);
    w.w = pack_bf16(b.z * p.scale, b.w * p.scale);
    *reinterpret_cast<uint4*>(p.dq + static_cast<size_t>(row) * p.d + c8 * 8) = w;
  }
}

// ------------------------------------------------------------ main kernel (B2)
template <int D>
struct BwdCfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int BM = 128;                      // query rows per step
  static constexpr int BN = 128;                      // keys per CTA
  static constexpr int STAGES = (D == 64) ? 2 : 1;
  static constexpr int CHUNKS = D / 64;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int VEC_BYTES = 512;               // 128 fp32
  // Q, dO, LSE2, D (+ padding to keep the next stage's tiles 1024-byte aligned)
  static constexpr int STAGE_STRIDE = 2 * TILE_BYTES + 1024;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE_BYTES;
  static constexpr int OFF_ST = 2 * TILE_BYTES;                              // + s * STAGE_STRIDE
  static constexpr int ST_Q = 0, ST_DO = TILE_BYTES, ST_LSE = 2 * TILE_BYTES, ST_D = 2 * TILE_BYTES + VEC_BYTES;
  static constexpr int OFF_PT = OFF_ST + STAGES * STAGE_STRIDE;             // 128 x 128 bf16
  static constexpr int OFF_DST = OFF_PT + 32768;
  static constexpr int OFF_BAR = OFF_DST + 32768;
  // kv_full, st_full[S], st_empty[S], s_full, dp_full, ds_ready, pds_free,
  // dq_full, dq_empty, dkv_done, drain
  static constexpr int NUM_BARS = 1 + 2 * STAGES + 8;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
  // d = 128 has no room left: dQ reuses the dP^T columns once dS is in smem
  static constexpr bool DQ_IN_DP = (D == 128);
  static constexpr uint32_t COL_DQ = DQ_IN_DP ? COL_DP : 256 + 2 * D;
};

struct BwdParams {
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dq_acc;       // [BH][Np][d]
  const float* lse2;   // [BH][Np]
  const float* delta;  // [BH][Np]
  int N;
  int Np;
  int n_ktiles;
  int causal;
  float scale;
  float scale_log2;
};

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

// Byte offset of 16-byte unit u (0..15) of row r in a [128][128] bf16 tile
// stored as two K-major 128-byte-swizzled halves of 64 columns.
__device__ __forceinline__ uint32_t sw128_offset(int r, int u) {
  return static_cast<uint32_t>((u >> 3) * 16384 + r * 128 + (((u & 7) ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    fa2_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ktile = blockIdx.x;  // causal: low key blocks see the most query blocks; run them first
  const int bh = blockIdx.y;
  const int k0 = ktile * C::BN;
  const int n_qtiles = p.n_ktiles;  // self-attention: same N
  const int i_first = p.causal ? ktile : 0;
  const int n_iter = n_qtiles - i_first;

  const uint32_t bar_kv = sbase + C::OFF_BAR;
  auto bar_st_full = [&](int s) { return sbase + C::OFF_BAR + 8 * (1 + s); };
  auto bar_st_empty = [&](int s) { return sbase + C::OFF_BAR + 8 * (1 + C::STAGES + s); };
  const uint32_t bar_s_full = sbase + C::OFF_BAR + 8 * (1 + 2 * C::STAGES);
  const uint32_t bar_dp_full = bar_s_full + 8;
  const uint32_t bar_ds_ready = bar_s_full + 16;
  const uint32_t bar_pds_free = bar_s_full + 24;
  const uint32_t bar_dq_full = bar_s_full + 32;
  const uint32_t bar_dq_empty = bar_s_full + 40;
  const uint32_t bar_dkv_done = bar_s_full + 48;
  const uint32_t bar_drain = bar_s_full + 56;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_st_full(s), 1);
      mbar_init(bar_st_empty(s), 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_ds_ready, 128);
    mbar_init(bar_pds_free, 1);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dq_empty, 128);
    mbar_init(bar_dkv_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_kv, 2 * C::TILE_BYTES);
      for (int c = 0; c < C::CHUNKS; ++c) {
        tma_load_3d(sbase + C::OFF_K + c * C::CHUNK_BYTES, &tm_k, bar_kv, c * 64, k0, bh);
        tma_load_3d(sbase + C::OFF_V + c * C::CHUNK_BYTES, &tm_v, bar_kv, c * 64, k0, bh);
      }
      int last_parity[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      for (int it = 0; it < n_iter && ok; ++it) {
        const int i = i_first + it;
        const int s = it % C::STAGES;
        const int n = it / C::STAGES;
        if (n > 0) ok = mbar_wait(bar_st_empty(s), (n - 1) & 1, abort_flag, 0x1101);
        if (!ok) break;
        const uint32_t st = sbase + C::OFF_ST + s * C::STAGE_STRIDE;
        const uint32_t bar = bar_st_full(s);
        mbar_arrive_expect_tx(bar, 2 * C::TILE_BYTES + 2 * C::VEC_BYTES);
        for (int c = 0; c < C::CHUNKS; ++c) {
          tma_load_3d(st + C::ST_Q + c * C::CHUNK_BYTES, &tm_q, bar, c * 64, i * C::BM, bh);
          tma_load_3d(st + C::ST_DO + c * C::CHUNK_BYTES, &tm_do, bar, c * 64, i * C::BM, bh);
        }
        const size_t voff = static_cast<size_t>(bh) * p.Np + static_cast<size_t>(i) * C::BM;
        bulk_load(st + C::ST_LSE, p.lse2 + voff, C::VEC_BYTES, bar);
        bulk_load(st + C::ST_D, p.delta + voff, C::VEC_BYTES, bar);
        last_parity[s] = n & 1;
      }
      mbar_wait(bar_kv, 0, abort_flag, 0x1102);
      for (int s = 0; s < C::STAGES; ++s)
        if (last_parity[s] >= 0) mbar_wait(bar_st_full(s), last_parity[s], abort_flag, 0x1103);
    }
  } else if (warp == 5) {
    // --------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_SS = idesc_bf16(128, 128, false, false);   // S^T, dP^T
      constexpr uint32_t IDESC_KV = idesc_bf16(128, D, false, true);      // dV, dK
      constexpr uint32_t IDESC_Q = idesc_bf16(128, D, true, true);        // dQ
      bool ok = mbar_wait(bar_kv, 0, abort_flag, 0x1201);
      for (int it = 0; it < n_iter && ok; ++it) {
        const int s = it % C::STAGES;
        const uint32_t st = sbase + C::OFF_ST + s * C::STAGE_STRIDE;
        ok = mbar_wait(bar_st_full(s), (it / C::STAGES) & 1, abort_flag, 0x1202);
        if (!ok) break;
        tc_fence_after();
        // S^T = K Q_i^T (the S columns were read before ds_ready(it-1), waited below)
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * C::CHUNK_BYTES + (k & 3) * 32;
          umma_ss(tmem + C::COL_S, sdesc_sw128(sbase + C::OFF_K + off, 16, 1024),
                  sdesc_sw128(st + C::ST_Q + off, 16, 1024), IDESC_SS, k > 0 ? 1u : 0u);
        }
        umma_commit(bar_s_full);
        // dP^T = V dO_i^T; with d = 128 the dP columns hold dQ_{i-1} until drained
        if (C::DQ_IN_DP && it > 0) {
          ok = mbar_wait(bar_dq_empty, (it - 1) & 1, abort_flag, 0x1203);
          if (!ok) break;
          tc_fence_after();
        }
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * C::CHUNK_BYTES + (k & 3) * 32;
          umma_ss(tmem + C::COL_DP, sdesc_sw128(sbase + C::OFF_V + off, 16, 1024),
                  sdesc_sw128(st + C::ST_DO + off, 16, 1024), IDESC_SS, k > 0 ? 1u : 0u);
        }
        umma_commit(bar_dp_full);
        // P^T and dS^T are in shared memory; S^T and dP^T have been read
        ok = mbar_wait(bar_ds_ready, it & 1, abort_flag, 0x1204);
        if (!ok) break;
        tc_fence_after();
        const uint32_t pt = sbase + C::OFF_PT;
        const uint32_t dst = sbase + C::OFF_DST;
#pragma unroll
        for (int k = 0; k < C::BM / 16; ++k) {
          const uint32_t aoff = (k >> 2) * C::CHUNK_BYTES + (k & 3) * 32;   // K-major over queries
          const uint64_t bdo = sdesc_sw128(st + C::ST_DO + k * 2048, C::CHUNK_BYTES, 1024);
          umma_ss(tmem + C::COL_DV, sdesc_sw128(pt + aoff, 16, 1024), bdo, IDESC_KV,
                  (it > 0 || k > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int k = 0; k < C::BM / 16; ++k) {
          const uint32_t aoff = (k >> 2) * C::CHUNK_BYTES + (k & 3) * 32;
          const uint64_t bq = sdesc_sw128(st + C::ST_Q + k * 2048, C::CHUNK_BYTES, 1024);
          umma_ss(tmem + C::COL_DK, sdesc_sw128(dst + aoff, 16, 1024), bq, IDESC_KV,
                  (it > 0 || k > 0) ? 1u : 0u);
        }
        if (!C::DQ_IN_DP && it > 0) {
          ok = mbar_wait(bar_dq_empty, (it - 1) & 1, abort_flag, 0x1205);
          if (!ok) break;
          tc_fence_after();
        }
        // dQ_i = dS K_j: A = dS (queries x keys), the dS^T buffer read MN-major
#pragma unroll
        for (int k = 0; k < C::BN / 16; ++k) {
          const uint64_t a = sdesc_sw128(dst + k * 2048, C::CHUNK_BYTES, 1024);
          const uint64_t b = sdesc_sw128(sbase + C::OFF_K + k * 2048, C::CHUNK_BYTES, 1024);
          umma_ss(tmem + C::COL_DQ, a, b, IDESC_Q, k > 0 ? 1u : 0u);
        }
        umma_commit(bar_dq_full);
        umma_commit(bar_pds_free);
        umma_commit(bar_st_empty(s));
      }
      umma_commit(bar_dkv_done);
      umma_commit(bar_drain);
      mbar_wait(bar_drain, 0, abort_flag, 0x1206);
    }
  } else {
    // ------------------------------------------------- P / dS / dQ warps (0-3)
    const int r = threadIdx.x;  // key row of this CTA == TMEM lane (S^T, dP^T, dK, dV)
    const int key = k0 + r;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float c = p.scale_log2;
    uint8_t* pt_row = smem + C::OFF_PT;
    uint8_t* ds_row = smem + C::OFF_DST;
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      const int i = i_first + it;
      const int s = it % C::STAGES;
      const uint8_t* st = smem + C::OFF_ST + s * C::STAGE_STRIDE;
      const float* lse2 = reinterpret_cast<const float*>(st + C::ST_LSE);
      const float* dlt = reinterpret_cast<const float*>(st + C::ST_D);
      // LSE2 and D of this query block were written by the TMA (async proxy)
      ok = mbar_wait(bar_st_full(s), (it / C::STAGES) & 1, abort_flag, 0x1300);
      if (!ok) break;
      ok = mbar_wait(bar_s_full, it & 1, abort_flag, 0x1301);
      if (!ok) break;
      ok = mbar_wait(bar_dp_full, it & 1, abort_flag, 0x1302);
      if (!ok) break;
      // the previous step's MMAs have finished reading P^T and dS^T
      if (it > 0) {
        ok = mbar_wait(bar_pds_free, (it - 1) & 1, abort_flag, 0x1303);
        if (!ok) break;
      }
      tc_fence_after();
      const bool diag = p.causal && (i == ktile);
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {  // 32 query columns at a time
        float sv[32], dp[32];
        tmem_ld32(lane_base + C::COL_S + 32 * q, sv);
        tmem_ld32(lane_base + C::COL_DP + 32 * q, dp);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int col = 32 * q + e;
          float p0 = ex2(fmaf(sv[e], c, -lse2[col]));
          float p1 = ex2(fmaf(sv[e + 1], c, -lse2[col + 1]));
          if (diag) {  // query i*128+col may see key k0+r only if col >= r
            if (col < r) p0 = 0.f;
            if (col + 1 < r) p1 = 0.f;
          }
          const float d0 = p0 * (dp[e] - dlt[col]);
          const float d1 = p1 * (dp[e + 1] - dlt[col + 1]);
          pk[e / 2] = pack_bf16(p0, p1);
          dk[e / 2] = pack_bf16(d0, d1);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t off = sw128_offset(r, 4 * q + u);
          *reinterpret_cast<uint4*>(pt_row + off) = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          *reinterpret_cast<uint4*>(ds_row + off) = make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar_ds_ready);
      // dQ_i (query rows on TMEM lanes) -> fp32 accumulator
      ok = mbar_wait(bar_dq_full, it & 1, abort_flag, 0x1304);
      if (!ok) break;
      tc_fence_after();
      float* dq_row = p.dq_acc + (static_cast<size_t>(bh) * p.Np + static_cast<size_t>(i) * C::BM + r) * D;
#pragma unroll 1
      for (int q = 0; q < D / 32; ++q) {
        float v[32];
        tmem_ld32(lane_base + C::COL_DQ + 32 * q, v);
#pragma unroll
        for (int e = 0; e < 32; e += 4) red_add_v4(dq_row + 32 * q + e, v[e], v[e + 1], v[e + 2], v[e + 3]);
      }
      tc_fence_before();
      mbar_arrive(bar_dq_empty);
    }
    if (ok) ok = mbar_wait(bar_dkv_done, 0, abort_flag, 0x1305);
    if (ok) {
      tc_fence_after();
      const bool store = key < p.N;
      const size_t off = (static_cast<size_t>(bh) * p.N + key) * D;
#pragma unroll 1
      for (int q = 0; q < D / 32; ++q) {
        float v[32];
        uint4 w[4];
        uint32_t* wu = reinterpret_cast<uint32_t*>(w);
        tmem_ld32(lane_base + C::COL_DV + 32 * q, v);
#pragma unroll
        for (int e = 0; e < 16; ++e) wu[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(p.dv + off + 32 * q);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = w[e];
        }
        tmem_ld32(lane_base + C::COL_DK + 32 * q, v);
#pragma unroll
        for (int e = 0; e < 16; ++e) wu[e] = pack_bf16(v[2 * e] * p.scale, v[2 * e + 1] * p.scale);
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(p.dk + off + 32 * q);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = w[e];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace fa2
