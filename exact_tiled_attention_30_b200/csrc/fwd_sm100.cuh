// Forward kernel of exact tiled attention for sm_100a (B200).
//
// Method ("FlashAttention-2" summary page, How It Works items 1-3; "FlashAttention
// (v2)" glossary page, definition and mechanism paragraphs; reproduction page of
// the FlashAttention-2 paper, closing paragraph on causal blocks):
//   * one CTA per (query block of 128 rows, batch*head): the sequence itself is
//     split across CTAs, not just batch and heads;
//   * K/V tiles of 128 keys stream through shared memory; the running row max m
//     and row sum l (online softmax) keep the N x N scores on chip;
//   * the accumulator is rescaled only when the running max grows, and divided
//     by l once, in the epilogue;
//   * causal: key tiles wholly above the diagonal are never visited and only
//     the diagonal tile is masked elementwise.
//
// B200 mapping (the pages' A100/H100 tiling is prior art only):
//   warp 4       TMA producer: Q once, then K_j/V_j into a STAGES-deep ring
//   warp 5       MMA issuer + TMEM owner: S_j = Q K_j^T (tcgen05, smem x smem ->
//                TMEM, double-buffered), O += P_j V_j (P from TMEM, V from smem)
//   warps 0-3    softmax: thread t owns query row t (= TMEM lane t); reads S_j
//                with tcgen05.ld, updates m and l, rescales O in TMEM when the
//                max grew, writes P_j as bf16 into TMEM; finally O/l and LSE.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O [256,256+D),
// P [384,448) as bf16 pairs. Scores are kept in base 2: c = scale * log2(e)
// folds the softmax scale into the exponent, m is stored pre-multiplied by c.
#pragma once

#include "sm100_ptx.cuh"

namespace fa2 {

template <int D>
struct FwdCfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int STAGES = (D == 64) ? 3 : 2;
  static constexpr int CHUNKS = D / 64;               // 128-byte swizzle atoms across d
  static constexpr int TILE_BYTES = BM * D * 2;       // one Q, K or V tile
  static constexpr int CHUNK_BYTES = 128 * 128;       // one [128 rows][64] bf16 box
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = TILE_BYTES;                           // + s * 2 * TILE_BYTES
  static constexpr int OFF_V = 2 * TILE_BYTES;                       // + s * 2 * TILE_BYTES
  static constexpr int OFF_BAR = TILE_BYTES * (1 + 2 * STAGES);
  // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_full, o_done, drain
  static constexpr int NUM_BARS = 1 + 2 * STAGES + 2 + 3;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;  // tmem slot, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  // ask for more than half an SM's shared memory so one CTA owns the TMEM
  static constexpr int SMEM_ALLOC = (SMEM_BYTES + 1024 > 120 * 1024) ? SMEM_BYTES + 1024 : 120 * 1024;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O = 256, COL_P = 384;
};

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  int N;
  int H;
  int n_qtiles;
  int causal;
  float scale_log2;  // scale * log2(e)
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    fa2_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qtile = p.n_qtiles - 1 - static_cast<int>(blockIdx.x);  // heaviest causal tiles first
  const int bh = blockIdx.y;
  const int q0 = qtile * C::BM;
  const int n_kv_total = (p.N + C::BN - 1) / C::BN;
  const int n_kv = p.causal ? min(n_kv_total, qtile + 1) : n_kv_total;

  const uint32_t bar_q = sbase + C::OFF_BAR;
  auto bar_kv_full = [&](int s) { return sbase + C::OFF_BAR + 8 * (1 + s); };
  auto bar_kv_empty = [&](int s) { return sbase + C::OFF_BAR + 8 * (1 + C::STAGES + s); };
  auto bar_s_full = [&](int b) { return sbase + C::OFF_BAR + 8 * (1 + 2 * C::STAGES + b); };
  const uint32_t bar_p_full = sbase + C::OFF_BAR + 8 * (3 + 2 * C::STAGES);
  const uint32_t bar_o_done = sbase + C::OFF_BAR + 8 * (4 + 2 * C::STAGES);
  const uint32_t bar_drain = sbase + C::OFF_BAR + 8 * (5 + 2 * C::STAGES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_kv_full(s), 1);
      mbar_init(bar_kv_empty(s), 1);
    }
    mbar_init(bar_s_full(0), 1);
    mbar_init(bar_s_full(1), 1);
    mbar_init(bar_p_full, 128);
    mbar_init(bar_o_done, 1);
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
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, C::TILE_BYTES);
      for (int c = 0; c < C::CHUNKS; ++c)
        tma_load_3d(sbase + C::OFF_Q + c * C::CHUNK_BYTES, &tm_q, bar_q, c * 64, q0, bh);
      int last_parity[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        const int s = j % C::STAGES;
        const int n = j / C::STAGES;
        if (n > 0) ok = mbar_wait(bar_kv_empty(s), (n - 1) & 1, abort_flag, 0x101);
        if (!ok) break;
        const uint32_t kdst = sbase + C::OFF_K + s * 2 * C::TILE_BYTES;
        const uint32_t vdst = sbase + C::OFF_V + s * 2 * C::TILE_BYTES;
        mbar_arrive_expect_tx(bar_kv_full(s), 2 * C::TILE_BYTES);
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_3d(kdst + c * C::CHUNK_BYTES, &tm_k, bar_kv_full(s), c * 64, j * C::BN, bh);
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_3d(vdst + c * C::CHUNK_BYTES, &tm_v, bar_kv_full(s), c * 64, j * C::BN, bh);
        last_parity[s] = n & 1;
      }
      // never leave the CTA with copies still landing in its shared memory
      mbar_wait(bar_q, 0, abort_flag, 0x102);
      for (int s = 0; s < C::STAGES; ++s)
        if (last_parity[s] >= 0) mbar_wait(bar_kv_full(s), last_parity[s], abort_flag, 0x103);
    }
  } else if (warp == 5) {
    // --------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(128, C::BN, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16(128, D, false, true);
      bool ok = mbar_wait(bar_q, 0, abort_flag, 0x201);
      auto issue_pv = [&](int t) -> bool {
        if (!mbar_wait(bar_p_full, t & 1, abort_flag, 0x202)) return false;
        tc_fence_after();
        const uint32_t vbase = sbase + C::OFF_V + (t % C::STAGES) * 2 * C::TILE_BYTES;
#pragma unroll
        for (int k = 0; k < C::BN / 16; ++k) {
          // V: MN-major (d contiguous), 16 keys = 2 swizzle atoms of 8 rows
          const uint64_t bdesc = sdesc_sw128(vbase + k * 16 * 128, C::CHUNK_BYTES, 1024);
          umma_ts(tmem + C::COL_O, tmem + C::COL_P + k * 8, bdesc, IDESC_O, (t > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(bar_o_done);
        umma_commit(bar_kv_empty(t % C::STAGES));
        return true;
      };
      for (int j = 0; j < n_kv && ok; ++j) {
        const int s = j % C::STAGES;
        const int b = j & 1;
        ok = mbar_wait(bar_kv_full(s), (j / C::STAGES) & 1, abort_flag, 0x203);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kbase = sbase + C::OFF_K + s * 2 * C::TILE_BYTES;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * C::CHUNK_BYTES + (k & 3) * 32;
          const uint64_t adesc = sdesc_sw128(sbase + C::OFF_Q + off, 16, 1024);
          const uint64_t bdesc = sdesc_sw128(kbase + off, 16, 1024);
          umma_ss(tmem + (b ? C::COL_S1 : C::COL_S0), adesc, bdesc, IDESC_S, k > 0 ? 1u : 0u);
        }
        umma_commit(bar_s_full(b));
        if (j > 0) ok = issue_pv(j - 1);
      }
      if (ok && n_kv > 0) issue_pv(n_kv - 1);
      // drain: every UMMA of this CTA has finished before TMEM is released
      umma_commit(bar_drain);
      mbar_wait(bar_drain, 0, abort_flag, 0x401);
    }
  } else {
    // ---------------------------------------------------------- softmax warps
    const int row = threadIdx.x;  // 0..127 == TMEM lane
    const int qrow = q0 + row;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float c = p.scale_log2;
    float m = -INFINITY;  // running max of c * s, base-2 units
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int b = j & 1;
      ok = mbar_wait(bar_s_full(b), (j >> 1) & 1, abort_flag, 0x301);
      if (!ok) break;
      tc_fence_after();
      const uint32_t scol = b ? C::COL_S1 : C::COL_S0;
      float s[128];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(lane_base + scol + 32 * q, *reinterpret_cast<float(*)[32]>(&s[32 * q]));
      const int k0 = j * C::BN;
      const bool need_mask = (p.causal && j == qtile) || (k0 + C::BN > p.N);
      if (need_mask) {
        const int lim = p.causal ? min(qrow + 1, p.N) : p.N;  // keys [0, lim) allowed
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (k0 + i >= lim) s[i] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int i = 1; i < 128; ++i) mx = fmaxf(mx, s[i]);
      const float m_new = fmaxf(m, mx * c);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2(m - m_use);
      float rs = 0.f;
      uint32_t pk[64];
      if (!need_mask) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float p0 = ex2(fmaf(s[2 * i], c, -m_use));
          const float p1 = ex2(fmaf(s[2 * i + 1], c, -m_use));
          rs += p0 + p1;
          pk[i] = pack_bf16(p0, p1);
        }
      } else {
        // masked keys contribute exactly 0 (also when c == 0, where -inf * c is NaN)
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float p0 = s[2 * i] == -INFINITY ? 0.f : ex2(fmaf(s[2 * i], c, -m_use));
          const float p1 = s[2 * i + 1] == -INFINITY ? 0.f : ex2(fmaf(s[2 * i + 1], c, -m_use));
          rs += p0 + p1;
          pk[i] = pack_bf16(p0, p1);
        }
      }
      l = l * alpha + rs;
      m = m_use;
      if (j > 0) {
        // PV_{j-1} must be done before O is rescaled and before P is overwritten
        ok = mbar_wait(bar_o_done, (j - 1) & 1, abort_flag, 0x302);
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int q = 0; q < D / 32; ++q) {
            float o[32];
            tmem_ld32(lane_base + C::COL_O + 32 * q, o);
            uint32_t u[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(o[i] * alpha);
            tmem_st32(lane_base + C::COL_O + 32 * q, u);
          }
        }
      }
      tmem_st32(lane_base + C::COL_P, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      tmem_st32(lane_base + C::COL_P + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p_full);
    }
    if (ok && n_kv > 0) ok = mbar_wait(bar_o_done, (n_kv - 1) & 1, abort_flag, 0x303);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool store = qrow < p.N;
      __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.N + qrow) * D;
#pragma unroll 1
      for (int q = 0; q < D / 32; ++q) {
        float o[32];
        tmem_ld32(lane_base + C::COL_O + 32 * q, o);
        uint4 w[4];
        uint32_t* wu = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int i = 0; i < 16; ++i) wu[i] = pack_bf16(o[2 * i] * inv_l, o[2 * i + 1] * inv_l);
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * q);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = w[i];
        }
      }
      if (store) p.lse[static_cast<size_t>(bh) * p.N + qrow] = (m + __log2f(l)) * 0.69314718055994530942f;
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace fa2
