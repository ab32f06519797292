// Forward kernel of exact tiled attention for sm_100a (B200).
//
// Method ("FlashAttention-2" summary page, How It Works items 1-3; "FlashAttention
// (v2)" glossary page, definition and mechanism paragraphs; reproduction page of
// the FlashAttention-2 paper, closing paragraph on causal blocks):
//   * the sequence is split across CTAs, not just batch and heads: one CTA per
//     (256-row query block, batch*head);
//   * K/V tiles of 128 keys stream through shared memory; the running row max m
//     and row sum l (online softmax) keep the N x N scores on chip;
//   * the accumulator is divided by l once, in the epilogue;
//   * causal: key tiles wholly above the diagonal are never visited and only
//     the diagonal tile of each query tile is masked elementwise.
//
// B200 mapping (the pages' A100/H100 tiling is prior art only):
//   warp 16       TMA producer: Q0, Q1 once, then K_j/V_j into a STAGES-deep ring
//   warp 17       MMA issuer + TMEM owner. Per key tile j it issues
//                 PV0_j, S0_{j+1}, PV1_j, S1_{j+1} (in that order), so while one
//                 tile's softmax runs the tensor core works on the other tile:
//                 S_t = Q_t K_j^T (smem x smem -> TMEM) and O_t += P_t V_j (P from
//                 TMEM, V from smem). The single issue order also keeps the two
//                 tiles' softmax phases apart (measured: one issuer per tile let
//                 them drift into step and contend for the MUFU unit).
//   warps 0-7     softmax of query tile 0, warps 8-15 of query tile 1. Two
//                 warpgroups per tile split each row: warpgroup h owns keys
//                 [64h, 64h+64) of row r (TMEM lane r): tcgen05.ld of its 64
//                 scores, partial row max (exchanged with the other half through
//                 shared memory, so both use one reference max), exp2, partial
//                 row sums, P written back as bf16 over the first 32 of its S
//                 columns. Halving the per-thread row shortens the softmax step
//                 that sits between the two MMAs of a tile.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D),
// O1 [256+D, 256+2D). Scores are kept in base 2: c = scale * log2(e) folds the
// softmax scale into the exponent and m is stored pre-multiplied by c.
//
// Rescaling: a row's reference max m only moves when the new tile's max exceeds
// it by more than 8 (base-2 units). Otherwise P keeps using the old m (entries
// up to 2^8, exact in fp32 accumulation and bf16's relative precision) and O is
// not touched. The result is unchanged because O and l share the same m and O/l
// is formed once at the end; LSE = m + log2(l) uses that same m. O is divided
// by the sum of the bf16-rounded weights it was accumulated with, so it stays
// a convex combination of V rows when one weight dominates; LSE uses the fp32 sum.
#pragma once

#include "exp2_poly.cuh"
#include "sm100_ptx.cuh"

namespace fa2 {

template <int D>
struct FwdCfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int BM = 128;                      // rows per query tile (two per CTA)
  static constexpr int BN = 128;                      // keys per K/V tile
  static constexpr int STAGES = (D == 64) ? 4 : 2;
  static constexpr int CHUNKS = D / 64;               // 128-byte swizzle atoms across d
  static constexpr int TILE_BYTES = BM * D * 2;       // one Q, K or V tile
  static constexpr int CHUNK_BYTES = 128 * 128;       // one [128 rows][64] bf16 box
  static constexpr int OFF_Q = 0;                     // Q0, Q1
  static constexpr int OFF_K = 2 * TILE_BYTES;        // + s * 2 * TILE_BYTES
  static constexpr int OFF_V = 3 * TILE_BYTES;        // + s * 2 * TILE_BYTES
  static constexpr int OFF_BAR = TILE_BYTES * (2 + 2 * STAGES);
  // q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done[2], drain,
  // xmax[2 tiles][2 slots], xsum[2 tiles]
  static constexpr int NUM_BARS = 1 + 2 * STAGES + 7 + 6;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;  // tmem slot, abort flag
  // exchange between the two halves of a row: partial maxima [tile][slot][half][row]
  // and, at the end, partial sums [tile][half][l | lr][row]
  static constexpr int OFF_XMAX = OFF_MISC + 16;
  static constexpr int OFF_XSUM = OFF_XMAX + 2 * 2 * 2 * 128 * 4;
  static constexpr int SMEM_BYTES = OFF_XSUM + 2 * 2 * 2 * 128 * 4;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;     // slack for 1024-byte alignment
  static constexpr int WARP_TMA = 16, WARP_MMA = 17;
  static constexpr int THREADS = 32 * 18;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
  static constexpr float RESCALE_THRESHOLD = 8.0f;         // log2 of the largest P entry
  static constexpr int HEAD_GROUP = 16;                    // causal launch order, see below
  // d = 64: one pair of weights in POLY_EVERY is exponentiated on the FMA pipe
  // (the MUFU unit is the tighter limit there); d = 128: MUFU only (measured faster)
  static constexpr int POLY_EVERY = (D == 64) ? 3 : 1 << 20;
};

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  int N;
  int n_qtiles;  // ceil(N / 128)
  int n_pairs;   // ceil(n_qtiles / 2)
  int BH;
  int causal;
  float scale_log2;  // scale * log2(e)
};

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
    fa2_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Blocks launch in linear order. Non-causal: grid (pair, batch*head), so the
  // pairs of one head run together and share its K/V tiles in L2. Causal: a 1-D
  // grid in groups of HEAD_GROUP heads (their K/V stay in L2 while the group
  // runs); inside a group the heaviest pairs of every head start first.
  int pair, bh;
  if (!p.causal) {
    pair = blockIdx.x;
    bh = blockIdx.y;
  } else {
    const int group_blocks = C::HEAD_GROUP * p.n_pairs;
    const int grp = static_cast<int>(blockIdx.x) / group_blocks;
    const int r = static_cast<int>(blockIdx.x) - grp * group_blocks;
    const int heads = min(C::HEAD_GROUP, p.BH - grp * C::HEAD_GROUP);
    pair = p.n_pairs - 1 - r / heads;
    bh = grp * C::HEAD_GROUP + r % heads;
  }
  const int n_kv_total = (p.N + C::BN - 1) / C::BN;
  // query tiles 2*pair and 2*pair+1; with causal masking tile t sees key tiles [0, qt_t]
  const int qt0 = 2 * pair;
  const int qt1 = 2 * pair + 1;
  const int n0 = p.causal ? min(n_kv_total, qt0 + 1) : n_kv_total;
  const int n1 = p.causal ? min(n_kv_total, qt1 + 1) : n_kv_total;  // n1 >= n0
#ifdef FA2_TRACE
  const bool trace_cta = p.causal ? blockIdx.x == 7 : (blockIdx.x == 0 && blockIdx.y == 7);
#endif

  const uint32_t bar_q = sbase + C::OFF_BAR;
  auto bar_kv_full = [&](int s) { return sbase + C::OFF_BAR + 8 * (1 + s); };
  auto bar_kv_empty = [&](int s) { return sbase + C::OFF_BAR + 8 * (1 + C::STAGES + s); };
  const uint32_t bar_base = sbase + C::OFF_BAR + 8 * (1 + 2 * C::STAGES);
  auto bar_s_full = [&](int t) { return bar_base + 8 * t; };
  auto bar_p_full = [&](int t) { return bar_base + 16 + 8 * t; };
  auto bar_o_done = [&](int t) { return bar_base + 32 + 8 * t; };
  const uint32_t bar_drain = bar_base + 48;
  auto bar_xmax = [&](int t, int slot) { return bar_base + 56 + 16 * t + 8 * slot; };
  auto bar_xsum = [&](int t) { return bar_base + 88 + 8 * t; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_kv_full(s), 1);
      mbar_init(bar_kv_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s_full(t), 1);
      mbar_init(bar_p_full(t), 256);
      mbar_init(bar_o_done(t), 1);
      mbar_init(bar_xmax(t, 0), 256);
      mbar_init(bar_xmax(t, 1), 256);
      mbar_init(bar_xsum(t), 256);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::WARP_TMA && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::WARP_TMA) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, 2 * C::TILE_BYTES);
      for (int c = 0; c < C::CHUNKS; ++c) {
        tma_load_3d(sbase + C::OFF_Q + c * C::CHUNK_BYTES, &tm_q, bar_q, c * 64, qt0 * C::BM, bh);
        tma_load_3d(sbase + C::OFF_Q + C::TILE_BYTES + c * C::CHUNK_BYTES, &tm_q, bar_q, c * 64,
                    qt1 * C::BM, bh);
      }
      int last_parity[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      for (int j = 0; j < n1 && ok; ++j) {
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
  } else if (warp == C::WARP_MMA) {
    // --------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(128, C::BN, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16(128, D, false, true);
      // descriptor halves of every operand buffer, built once
      const SDesc dq0 = sdesc_make(sbase + C::OFF_Q, 16, 1024);
      const SDesc dq1 = sdesc_make(sbase + C::OFF_Q + C::TILE_BYTES, 16, 1024);
      const SDesc dk0 = sdesc_make(sbase + C::OFF_K, 16, 1024);
      const SDesc dv0 = sdesc_make(sbase + C::OFF_V, C::CHUNK_BYTES, 1024);
      constexpr uint32_t STAGE16 = 2 * C::TILE_BYTES / 16;  // stage stride in descriptor units
      auto issue_s = [&](int t, int j) {
        const uint32_t klo = dk0.lo + (j % C::STAGES) * STAGE16;
        const uint32_t qlo = t ? dq1.lo : dq0.lo;
        const uint32_t dcol = tmem + (t ? C::COL_S1 : C::COL_S0);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * C::CHUNK_BYTES + (k & 3) * 32) >> 4;
          umma_ss2(dcol, qlo + off, dq0.hi, klo + off, dk0.hi, IDESC_S, k > 0 ? 1u : 0u);
        }
        umma_commit(bar_s_full(t));
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t vlo = dv0.lo + (j % C::STAGES) * STAGE16;
        const uint32_t pcol = tmem + (t ? C::COL_S1 : C::COL_S0);
        const uint32_t ocol = tmem + (t ? C::COL_O1 : C::COL_O0);
        const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
        for (int k = 0; k < C::BN / 16; ++k) {
          // V: MN-major (d contiguous), 16 keys = 2 swizzle atoms of 8 rows. P of
          // keys [64h, 64h+64) sits in columns [64h, 64h+32)
          umma_ts2(ocol, pcol + k * 8 + (k >= 4 ? 32 : 0), vlo + k * (2048 >> 4), dv0.hi, IDESC_O,
                   k > 0 ? 1u : acc0);
        }
      };
      bool ok = mbar_wait(bar_q, 0, abort_flag, 0x201) &&
                mbar_wait(bar_kv_full(0), 0, abort_flag, 0x202);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
      }
      int kv_waited = 0;  // highest key tile whose kv_full has been waited for
      auto wait_kv = [&](int j) -> bool {
        if (j <= kv_waited) return true;
        kv_waited = j;
        if (!mbar_wait(bar_kv_full(j % C::STAGES), (j / C::STAGES) & 1, abort_flag, 0x203)) return false;
        tc_fence_after();
        return true;
      };
      for (int j = 0; j < n1 && ok; ++j) {
        if (j < n0) {
          ok = mbar_wait(bar_p_full(0), j & 1, abort_flag, 0x204);
          if (!ok) break;
          FA2_TRACE_AT(trace_cta, 16, j);
          tc_fence_after();
          issue_pv(0, j);
          if (j + 1 < n0) {
            ok = wait_kv(j + 1);
            if (!ok) break;
            issue_s(0, j + 1);  // overwrites S0/P0 after PV0_j in issue order
            FA2_TRACE_AT(trace_cta, 17, j);
          } else {
            umma_commit(bar_o_done(0));
          }
        }
        ok = mbar_wait(bar_p_full(1), j & 1, abort_flag, 0x205);
        if (!ok) break;
        FA2_TRACE_AT(trace_cta, 18, j);
        tc_fence_after();
        issue_pv(1, j);
        umma_commit(bar_kv_empty(j % C::STAGES));  // K_j and V_j fully consumed
        if (j + 1 < n1) {
          ok = wait_kv(j + 1);
          if (!ok) break;
          issue_s(1, j + 1);
          FA2_TRACE_AT(trace_cta, 19, j);
        } else {
          umma_commit(bar_o_done(1));
        }
      }
      // drain: every UMMA of this CTA has finished before TMEM is released
      umma_commit(bar_drain);
      mbar_wait(bar_drain, 0, abort_flag, 0x206);
    }
  } else {
    // ---------------------------------------------------------- softmax warps
    const int t = warp >> 3;              // query tile of this warpgroup
    const int h = (warp >> 2) & 1;        // key half: keys [64h, 64h+64) of each tile
    const int row = threadIdx.x & 127;    // TMEM lane
    const int qt = t ? qt1 : qt0;
    const int n_t = t ? n1 : n0;
    const int qrow = qt * C::BM + row;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t scol = (t ? C::COL_S1 : C::COL_S0) + 64 * h;  // this half's scores
    constexpr int DH = D / 2;                                    // O columns per half
    const uint32_t ocol = (t ? C::COL_O1 : C::COL_O0) + DH * h;
    float* xmax = reinterpret_cast<float*>(smem + C::OFF_XMAX) + t * 512 + row;  // + slot*256 + half*128
    float* xsum = reinterpret_cast<float*>(smem + C::OFF_XSUM) + t * 512 + row;  // + half*256 + which*128
    const float c = p.scale_log2;
    float m = -INFINITY;  // reference max of c * s, base-2 units (same in both halves)
    float l = 0.f;        // this half's row sum of the weights 2^(c s - m)
    float lr = 0.f;       // the same sum over the weights rounded to bf16
    bool ok = true;
#ifdef FA2_TRACE
    const bool trace_row = trace_cta && row == 0 && h == 0;
#endif
    for (int j = 0; j < n_t; ++j) {
      FA2_TRACE_AT(trace_row, 8 * t + 0, j);
      ok = mbar_wait(bar_s_full(t), j & 1, abort_flag, 0x301);
      if (!ok) break;
      FA2_TRACE_AT(trace_row, 8 * t + 1, j);
      tc_fence_after();
      const int k0 = j * C::BN + 64 * h;  // first key of this half
      const bool need_mask = (p.causal && j == qt) || (j * C::BN + C::BN > p.N);
      const int lim = p.causal ? min(qrow + 1, p.N) : p.N;  // keys [0, lim) allowed
      float s[64];
      tmem_ld64(lane_base + scol, s);
      if (need_mask) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (k0 + i >= lim) s[i] = -INFINITY;
      }
      float mx;
      {
        float a = s[0], b = s[1];
#pragma unroll
        for (int i = 2; i < 62; i += 4) {
          a = max3(a, s[i], s[i + 1]);
          b = max3(b, s[i + 2], s[i + 3]);
        }
        mx = max3(a, b, fmaxf(s[62], s[63]));
      }
      // row max over both halves: publish this half's, read the other's
      const int slot = j & 1;
      xmax[slot * 256 + h * 128] = mx;
      mbar_arrive(bar_xmax(t, slot));
      ok = mbar_wait(bar_xmax(t, slot), (j >> 1) & 1, abort_flag, 0x304);
      if (!ok) break;
      mx = fmaxf(mx, xmax[slot * 256 + (1 - h) * 128]);
      FA2_TRACE_AT(trace_row, 8 * t + 2, j);
      const float m_cand = fmaxf(m, mx * c);
      const bool grow = m_cand - m > C::RESCALE_THRESHOLD;  // always true for the first tile
      const float alpha = grow ? ex2(m - m_cand) : 1.f;
      if (grow) m = m_cand;
      // weights 2^(c s - m) in pairs, written back over this half's S as bf16 P.
      // rs: sum of the fp32 weights (for LSE); rr: sum of the bf16-rounded weights
      // that the P V product actually uses (for O / l, so O stays a convex
      // combination of V rows even when one weight dominates)
      const unsigned long long c2 = f2(c, c), negm2 = f2(-m, -m);
      unsigned long long rs2 = f2(0.f, 0.f), rr2 = f2(0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t pk[16];
        if (!need_mask) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = 32 * q + 2 * i;
            float x0, x1, p0, p1;
            f2_split(f2_fma(f2(s[e], s[e + 1]), c2, negm2), x0, x1);
            if ((16 * q + i) % C::POLY_EVERY == C::POLY_EVERY - 1) {
              exp2_poly2(x0, x1, p0, p1);  // FMA pipe: balances the MUFU unit
            } else {
              p0 = ex2(x0);
              p1 = ex2(x1);
            }
            const uint32_t w = pack_bf16(p0, p1);
            pk[i] = w;
            rs2 = f2_add(rs2, f2(p0, p1));
            rr2 = f2_add(rr2, f2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)));
          }
        } else {
          // masked keys contribute exactly 0 (also when c == 0, where -inf * c is NaN)
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = 32 * q + 2 * i;
            const float p0 = k0 + e >= lim ? 0.f : ex2(fmaf(s[e], c, -m));
            const float p1 = k0 + e + 1 >= lim ? 0.f : ex2(fmaf(s[e + 1], c, -m));
            const uint32_t w = pack_bf16(p0, p1);
            pk[i] = w;
            rs2 = f2_add(rs2, f2(p0, p1));
            rr2 = f2_add(rr2, f2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)));
          }
        }
        // P of keys [32q, 32q+32) of this half -> columns [16q, 16q+16): the scores
        // there are already in registers
        tmem_st16(lane_base + scol + 16 * q, pk);
      }
      FA2_TRACE_AT(trace_row, 8 * t + 3, j);
      float rs_lo, rs_hi, rr_lo, rr_hi;
      f2_split(rs2, rs_lo, rs_hi);
      f2_split(rr2, rr_lo, rr_hi);
      l = l * alpha + (rs_lo + rs_hi);
      lr = lr * alpha + (rr_lo + rr_hi);
      // O holds PV_0..PV_{j-1}: all complete, since S_j was issued after them.
      // Each half rescales its own D/2 columns of O.
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
        for (int q = 0; q < DH / 32; ++q) {
          float o[32];
          tmem_ld32(lane_base + ocol + 32 * q, o);
          uint32_t u[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(o[i] * alpha);
          tmem_st32(lane_base + ocol + 32 * q, u);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p_full(t));
      FA2_TRACE_AT(trace_row, 8 * t + 4, j);
    }
    if (ok && n_t > 0) ok = mbar_wait(bar_o_done(t), 0, abort_flag, 0x303);
    if (ok) {
      // row sums over both halves
      xsum[h * 256] = l;
      xsum[h * 256 + 128] = lr;
      mbar_arrive(bar_xsum(t));
      ok = mbar_wait(bar_xsum(t), 0, abort_flag, 0x305);
    }
    if (ok) {
      l += xsum[(1 - h) * 256];
      lr += xsum[(1 - h) * 256 + 128];
      tc_fence_after();
      const float inv_l = 1.f / lr;
      const bool store = qrow < p.N;
      __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.N + qrow) * D + DH * h;
#pragma unroll 1
      for (int q = 0; q < DH / 32; ++q) {
        float o[32];
        tmem_ld32(lane_base + ocol + 32 * q, o);
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
      if (store && h == 0)
        p.lse[static_cast<size_t>(bh) * p.N + qrow] = (m + __log2f(l)) * 0.69314718055994530942f;
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::WARP_MMA) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace fa2
