// Forward kernel of exact tiled attention for sm_100a (B200).
//
// Method ("FlashAttention-2" summary page, How It Works items 1-3; "FlashAttention
// (v2)" glossary page, definition and mechanism paragraphs; reproduction page of
// the FlashAttention-2 paper, closing paragraph on causal blocks):
//   * the sequence is split across CTAs, not just batch and heads: the work
//     items are (256-row query block, batch*head) pairs, taken by a persistent
//     grid of one CTA per SM from a work counter, heaviest first;
//   * K/V tiles of 128 keys stream through shared memory; the running row max m
//     and row sum l (online softmax) keep the N x N scores on chip;
//   * the accumulator is divided by l once, in the epilogue;
//   * causal: key tiles wholly above the diagonal are never visited and only
//     the diagonal tile of each query tile is masked elementwise (with Nq != Nk
//     the diagonal is that of the bottom-right corner: query i sees keys
//     j <= i + Nk - Nq).
//
// B200 mapping (the pages' A100/H100 tiling is prior art only):
//   warp 16       scheduler + TMA producer: takes the next item, hands it to the
//                 other warps through a two-slot ring, loads Q0, Q1 once the
//                 previous item's last S MMA is done, K_j/V_j into a STAGES-deep
//                 ring that continues across items
//   (warps 16 and 17 run converged: the whole warp executes the loop and
//   elect.sync inside each copy / MMA instruction picks the issuing lane)
//   warp 17       MMA issuer + TMEM owner. Per key tile j it issues
//                 PV0_j, S0_{j+1}, PV1_j, S1_{j+1} at d = 128 and PV0_j,
//                 S1_{j+1}, PV1_j, S0_{j+2} at d = 64 (three rotating S
//                 buffers), so while one tile's softmax runs the tensor core
//                 works on the other tile: S_t = Q_t K_j^T (smem x smem -> TMEM)
//                 and O_t += P_t V_j (P from TMEM, V from smem). The single issue
//                 order also keeps the two tiles' softmax phases apart (measured:
//                 one issuer per tile let them drift into step and contend for
//                 the MUFU unit). Non-causal d = 128 launches (EARLY) may issue
//                 the next item's first S0 while tile 1 forms its last P.
//   warps 0-7     softmax of query tile 0, warps 8-15 of query tile 1. Two
//                 warpgroups per tile split each row: warpgroup h owns keys
//                 [64h, 64h+64) of row r (TMEM lane r): tcgen05.ld of its 64
//                 scores, partial row max (exchanged with the other half through
//                 shared memory, so both use one reference max), exp2, partial
//                 row sums, P written back as bf16 over the first 32 of its S
//                 columns. Halving the per-thread row shortens the softmax step
//                 that sits between the two MMAs of a tile. Epilogue per item:
//                 O / l, stored with lanes transposed in groups so that every
//                 store instruction writes whole row segments; O is released to
//                 the next item's first PV as soon as it has been read.
// Tensor memory (512 columns): d = 128: S0 [0,128), S1 [128,256), O0 [256,384),
// O1 [384,512); d = 64: S buffers [0,128), [128,256), [256,384), O0 [384,448),
// O1 [448,512). Scores are kept in base 2: c = scale * log2(e) folds the
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
  // q_full, q_empty, kv_full[S], kv_empty[S], s_full[2 tiles][2], p_full[2][2],
  // o_done[2], o_free[2], drain, xmax[2 tiles][2 slots], xsum[2 tiles],
  // item_full[2], item_empty[2], pv_done[2]
  static constexpr int NUM_BARS = 2 + 2 * STAGES + 25;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;  // tmem slot, abort flag, items[2]
  // exchange between the two halves of a row: partial maxima [tile][slot][half][row]
  // and, at the end, partial sums [tile][half][l | lr][row]
  static constexpr int OFF_XMAX = OFF_MISC + 16;
  static constexpr int OFF_XSUM = OFF_XMAX + 2 * 2 * 2 * 128 * 4;
  static constexpr int SMEM_BYTES = OFF_XSUM + 2 * 2 * 2 * 128 * 4;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;     // slack for 1024-byte alignment
  static constexpr int WARP_TMA = 16, WARP_MMA = 17;
  static constexpr int THREADS = 32 * 18;
  static constexpr uint32_t TMEM_COLS = 512;
  // d = 64 has room for three S buffers that the two query tiles take in turn
  // (ROT, see the MMA issuer): S_t of the item's j-th key tile lives in buffer
  // (2 j + t) mod 3, so each tile's next S is computed while its softmax runs.
  // d = 128: one S buffer per tile.
  static constexpr bool ROT = (D == 64);
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128;
  static constexpr uint32_t COL_O0 = ROT ? 384 : 256, COL_O1 = ROT ? 448 : 256 + D;
  static constexpr float RESCALE_THRESHOLD = 8.0f;         // log2 of the largest P entry
  // d = 64: one pair of weights in POLY_EVERY is exponentiated on the FMA pipe
  // (the MUFU unit is the tighter limit there; one in 8 measured fastest of
  // 2, 3, 4, 5, 6, 8, 12 and none); d = 128: MUFU only (measured faster)
  static constexpr int POLY_EVERY = (D == 64) ? 8 : 1 << 20;
};

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  // work counter of this launch: both 32-bit halves hold `tag` at launch; the
  // high half keeps it (a different value means another launch has reset the
  // slot), the low half minus tag counts the items taken
  unsigned long long* counter;
  unsigned int tag;
  int Nq;        // query rows (O, LSE)
  int Nk;        // key rows
  int kq_offset; // Nk - Nq: causal query i sees keys j <= i + kq_offset
  int n_qtiles;  // ceil(Nq / 128)
  int n_pairs;   // ceil(n_qtiles / 2)
  int BH;
  int causal;
  int head_group;    // heads per causal scheduling group (see fwd_decode_item)
  float scale_log2;  // scale * log2(e)
};

// Work item -> (pair of query tiles, batch*head). Non-causal: the pairs of one
// head are consecutive, so they run together and share its K/V tiles in L2.
// Causal: groups of head_group heads (their K/V stay in L2 while the group
// runs; the host sizes the group to the L2); inside a group the heaviest pairs
// of every head come first.
__device__ __forceinline__ void fwd_decode_item(int item, int n_pairs, int BH, int head_group,
                                                bool causal, int& pair, int& bh) {
  if (!causal) {
    bh = item / n_pairs;
    pair = item - bh * n_pairs;
    return;
  }
  const int group_items = head_group * n_pairs;
  const int grp = item / group_items;
  const int r = item - grp * group_items;
  const int heads = min(head_group, BH - grp * head_group);
  pair = n_pairs - 1 - r / heads;
  bh = grp * head_group + r % heads;
}

// Persistent: one CTA per SM takes work items (pairs of query tiles) from a
// counter until none are left. Every barrier phase is counted over the CTA's
// whole sequence of items: `n` counts items, `kg` key tiles loaded, `jt[t]`
// key tiles of query tile t.
// EARLY (d = 128, items whose two tiles have equally many key tiles, i.e.
// non-causal launches): the next item's first S0 may be issued while the
// current item's tile 1 forms its last P (see the MMA issuer). A separate
// instantiation, so that causal launches run the plain schedule's code.
template <int D, bool EARLY = false>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
    fa2_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = p.n_pairs * p.BH;
  const int n_kv_total = (p.Nk + C::BN - 1) / C::BN;
  // query tiles 2*pair and 2*pair+1; with causal masking the last row of tile qt
  // sees keys up to qt*128 + 127 + kq_offset (self-attention: key tiles [0, qt])
  auto tiles_of = [&](int pair, int& n0, int& n1) {
    n0 = p.causal ? min(n_kv_total, (2 * pair * C::BM + C::BM - 1 + p.kq_offset) / C::BN + 1) : n_kv_total;
    n1 = p.causal ? min(n_kv_total, ((2 * pair + 1) * C::BM + C::BM - 1 + p.kq_offset) / C::BN + 1)
                  : n_kv_total;  // n0 <= n1 <= n0 + 1
  };
#ifdef FA2_TRACE
  const bool trace_cta = blockIdx.x == 7;
#endif

  const uint32_t bar_q_full = sbase + C::OFF_BAR;
  const uint32_t bar_q_empty = bar_q_full + 8;
  auto bar_kv_full = [&](int s) { return sbase + C::OFF_BAR + 8 * (2 + s); };
  auto bar_kv_empty = [&](int s) { return sbase + C::OFF_BAR + 8 * (2 + C::STAGES + s); };
  const uint32_t bar_base = sbase + C::OFF_BAR + 8 * (2 + 2 * C::STAGES);
  // s_full / p_full: d = 128 uses barrier 0 of each tile (phase = the tile's key
  // tile count); d = 64 alternates barriers 0 and 1 (phase = count / 2), since
  // its S runs two key tiles ahead of the softmax.
  auto bar_s_full = [&](int t, int k) { return bar_base + 8 * (2 * t + k); };
  auto bar_p_full = [&](int t, int k) { return bar_base + 32 + 8 * (2 * t + k); };
  auto bar_o_done = [&](int t) { return bar_base + 64 + 8 * t; };
  auto bar_o_free = [&](int t) { return bar_base + 80 + 8 * t; };
  const uint32_t bar_drain = bar_base + 96;
  auto bar_xmax = [&](int t, int slot) { return bar_base + 104 + 16 * t + 8 * slot; };
  auto bar_xsum = [&](int t) { return bar_base + 136 + 8 * t; };
  auto bar_item_full = [&](int q) { return bar_base + 152 + 8 * q; };
  auto bar_item_empty = [&](int q) { return bar_base + 168 + 8 * q; };
  auto bar_pv_done = [&](int t) { return bar_base + 184 + 8 * t; };  // d = 64: one phase per P V
  // barrier index and phase parity of the g-th key tile of a query tile
  auto sp_k = [&](int g) { return C::ROT ? (g & 1) : 0; };
  auto sp_par = [&](int g) { return static_cast<uint32_t>(C::ROT ? ((g >> 1) & 1) : (g & 1)); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);  // [2]

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_kv_full(s), 1);
      mbar_init(bar_kv_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      for (int k = 0; k < 2; ++k) {
        mbar_init(bar_s_full(t, k), 1);
        mbar_init(bar_p_full(t, k), 256);
      }
      mbar_init(bar_pv_done(t), 1);
      mbar_init(bar_o_done(t), 1);
      mbar_init(bar_o_free(t), 256);
      mbar_init(bar_xmax(t, 0), 256);
      mbar_init(bar_xmax(t, 1), 256);
      mbar_init(bar_xsum(t), 256);
    }
    mbar_init(bar_drain, 1);
    for (int q = 0; q < 2; ++q) {
      mbar_init(bar_item_full(q), 1);
      mbar_init(bar_item_empty(q), 1 + 512);  // MMA thread + softmax threads
    }
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

  // Consumers read item n from the two-slot ring (-1 ends the sequence).
  auto take_item = [&](int n, int site) -> int {
    if (!mbar_wait(bar_item_full(n & 1), (n >> 1) & 1, abort_flag, site)) return -1;
    const int item = item_slot[n & 1];
    mbar_arrive(bar_item_empty(n & 1));
    return item;
  };
  // the same for the converged MMA warp, which counts as one consumer
  auto take_item_w = [&](int n, int site) -> int {
    if (!mbar_wait_all(bar_item_full(n & 1), (n >> 1) & 1, abort_flag, site)) return -1;
    const int item = item_slot[n & 1];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_item_empty(n & 1));
    return item;
  };

  if (warp == C::WARP_TMA) {
    // ------------------------------------------------- scheduler + TMA producer
    // The whole warp runs this loop converged; elect.sync inside each copy and
    // expect_tx picks the issuing lane (see umma_ss2_w).
    {
      int last_parity[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) last_parity[s] = -1;
      int last_q_parity = -1;
      bool ok = true;
      int kg = 0;  // key tiles loaded so far
      for (int n = 0; ok; ++n) {
        int item = -1;
        if (lane == 0) {
          const unsigned long long v = atomicAdd(p.counter, 1ull);
          if (static_cast<unsigned int>(v >> 32) != p.tag) {
            report_conflict(0x10A);  // the slot now belongs to another launch: stop
          } else {
            const unsigned int taken = static_cast<unsigned int>(v) - p.tag;
            if (taken < static_cast<unsigned int>(n_items)) item = static_cast<int>(taken);
          }
        }
        item = __shfl_sync(0xffffffffu, item, 0);
        if (n >= 2) ok = mbar_wait_all(bar_item_empty(n & 1), ((n >> 1) - 1) & 1, abort_flag, 0x104);
        if (!ok) break;
        if (lane == 0) {
          item_slot[n & 1] = item;
          mbar_arrive(bar_item_full(n & 1));
        }
        __syncwarp();
        if (item < 0) break;
        int pair, bh, n0, n1;
        fwd_decode_item(item, p.n_pairs, p.BH, p.head_group, p.causal != 0, pair, bh);
        tiles_of(pair, n0, n1);
        // Q0, Q1 once the previous item's S MMAs are done with the buffers
        if (n >= 1) ok = mbar_wait_all(bar_q_empty, (n - 1) & 1, abort_flag, 0x105);
        if (!ok) break;
        mbar_arrive_expect_tx_w(bar_q_full, 2 * C::TILE_BYTES);
        for (int c = 0; c < C::CHUNKS; ++c) {
          tma_load_3d_w(sbase + C::OFF_Q + c * C::CHUNK_BYTES, &tm_q, bar_q_full, c * 64,
                      2 * pair * C::BM, bh);
          tma_load_3d_w(sbase + C::OFF_Q + C::TILE_BYTES + c * C::CHUNK_BYTES, &tm_q, bar_q_full,
                      c * 64, (2 * pair + 1) * C::BM, bh);
        }
        last_q_parity = n & 1;
        for (int j = 0; j < n1 && ok; ++j, ++kg) {
          const int s = kg % C::STAGES;
          const int u = kg / C::STAGES;
          if (u > 0) ok = mbar_wait_all(bar_kv_empty(s), (u - 1) & 1, abort_flag, 0x101);
          if (!ok) break;
#ifdef FA2_TEST_HOOKS
          if (g_test_stall_kv > 0 && kg + 1 == g_test_stall_kv) continue;  // planted stall
#endif
          const uint32_t kdst = sbase + C::OFF_K + s * 2 * C::TILE_BYTES;
          const uint32_t vdst = sbase + C::OFF_V + s * 2 * C::TILE_BYTES;
          mbar_arrive_expect_tx_w(bar_kv_full(s), 2 * C::TILE_BYTES);
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_3d_w(kdst + c * C::CHUNK_BYTES, &tm_k, bar_kv_full(s), c * 64, j * C::BN, bh);
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_3d_w(vdst + c * C::CHUNK_BYTES, &tm_v, bar_kv_full(s), c * 64, j * C::BN, bh);
          last_parity[s] = u & 1;
        }
      }
      // never leave the CTA with copies still landing in its shared memory
      if (last_q_parity >= 0) mbar_drain_wait(bar_q_full, last_q_parity, 0x102);
      for (int s = 0; s < C::STAGES; ++s)
        if (last_parity[s] >= 0) mbar_drain_wait(bar_kv_full(s), last_parity[s], 0x103);
    }
  } else if (warp == C::WARP_MMA) {
    // --------------------------------------------------------------- MMA issuer
    // The whole warp runs this loop converged; elect.sync inside each MMA and
    // commit picks the issuing lane (see umma_ss2_w).
    {
      constexpr uint32_t IDESC_S = idesc_bf16(128, C::BN, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16(128, D, false, true);
      // descriptor halves of every operand buffer, built once
      const SDesc dq0 = sdesc_make(sbase + C::OFF_Q, 16, 1024);
      const SDesc dq1 = sdesc_make(sbase + C::OFF_Q + C::TILE_BYTES, 16, 1024);
      const SDesc dk0 = sdesc_make(sbase + C::OFF_K, 16, 1024);
      const SDesc dv0 = sdesc_make(sbase + C::OFF_V, C::CHUNK_BYTES, 1024);
      constexpr uint32_t STAGE16 = 2 * C::TILE_BYTES / 16;  // stage stride in descriptor units
      // S buffer of tile t's j-th key tile of the current item
      auto sbuf = [&](int t, int j) -> uint32_t {
        if constexpr (C::ROT) return static_cast<uint32_t>((2 * j + t) % 3) * 128u;
        return t ? C::COL_S1 : C::COL_S0;
      };
      int jt0 = 0, jt1 = 0;   // key tiles of query tile 0 / 1 so far (s_full, p_full phases)
      // S_t of the item's key tile j, from the K/V ring slot of key tile g
      // (counted over the CTA's items)
      auto issue_s = [&](int t, int j, int g) {
        const uint32_t klo = dk0.lo + (g % C::STAGES) * STAGE16;
        const uint32_t qlo = t ? dq1.lo : dq0.lo;
        const uint32_t dcol = tmem + sbuf(t, j);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * C::CHUNK_BYTES + (k & 3) * 32) >> 4;
          umma_ss2_w(dcol, qlo + off, dq0.hi, klo + off, dk0.hi, IDESC_S, k > 0 ? 1u : 0u);
        }
        const int gt = (t ? jt1 : jt0) + j;
        umma_commit_w(bar_s_full(t, sp_k(gt)));
      };
      auto issue_pv = [&](int t, int j, int g, bool acc) {
        const uint32_t vlo = dv0.lo + (g % C::STAGES) * STAGE16;
        const uint32_t pcol = tmem + sbuf(t, j);
        const uint32_t ocol = tmem + (t ? C::COL_O1 : C::COL_O0);
        const uint32_t acc0 = acc ? 1u : 0u;
#pragma unroll
        for (int k = 0; k < C::BN / 16; ++k) {
          // V: MN-major (d contiguous), 16 keys = 2 swizzle atoms of 8 rows. P of
          // keys [64h, 64h+64) sits in columns [64h, 64h+32)
          umma_ts2_w(ocol, pcol + k * 8 + (k >= 4 ? 32 : 0), vlo + k * (2048 >> 4), dv0.hi, IDESC_O,
                   k > 0 ? 1u : acc0);
        }
        if constexpr (C::ROT) umma_commit_w(bar_pv_done(t));
      };
      auto wait_p = [&](int t, int j, unsigned int site) {
        const int gt = (t ? jt1 : jt0) + j;
        return mbar_wait_all(bar_p_full(t, sp_k(gt)), sp_par(gt), abort_flag, site);
      };
      bool ok = true;
      int kg = 0;             // key tiles consumed so far (K/V ring position)
      int kv_waited = -1;     // highest key tile (counted like kg) whose kv_full was waited for
      auto wait_kv = [&](int g) -> bool {
        if (g <= kv_waited) return true;
        kv_waited = g;
        if (!mbar_wait_all(bar_kv_full(g % C::STAGES), (g / C::STAGES) & 1, abort_flag, 0x203)) return false;
        tc_fence_after();
        return true;
      };
      // d = 128: the next item, taken and its first S0 issued while the current
      // item's tile 1 is still on its last key tile (see below)
      int next_item = -2;      // -2: not taken yet
      bool s0_early = false;   // the current item's S0 of key tile 0 is issued
      for (int n = 0; ok; ++n) {
        int item;
        if (next_item != -2) {
          item = next_item;
          next_item = -2;
        } else {
          item = take_item_w(n, 0x207);
        }
        if (item < 0) break;
        int pair, bh, n0, n1;
        fwd_decode_item(item, p.n_pairs, p.BH, p.head_group, p.causal != 0, pair, bh);
        tiles_of(pair, n0, n1);
        FA2_TRACE_AT(trace_cta, 20, n);
        if (!s0_early) {
          ok = mbar_wait_all(bar_q_full, n & 1, abort_flag, 0x201) && wait_kv(kg);
          if (!ok) break;
        }
        FA2_TRACE_AT(trace_cta, 21, n);
        tc_fence_after();
        // S of the item's first key tile: the S columns were last read by the
        // previous item's PV, which this thread issued before
        if (!s0_early) issue_s(0, 0, kg);
        s0_early = false;
        issue_s(1, 0, kg);
        if (n1 == 1) umma_commit_w(bar_q_empty);  // every S of the item issued
        if constexpr (C::ROT) {
          // Three S buffers: tile 0's S runs two key tiles ahead (S0_{j+2} takes
          // the buffer P1_j leaves), tile 1's one (S1_{j+1} takes the buffer P0_j
          // leaves), so both softmaxes find their next S ready when they finish.
          // Issue order per key tile j: PV0_j, S1_{j+1}, PV1_j, S0_{j+2}.
          if (n0 > 1) {
            ok = wait_kv(kg + 1);
            if (!ok) break;
            issue_s(0, 1, kg + 1);
          }
          for (int j = 0; j < n1 && ok; ++j) {
            const int g = kg + j;
            if (j < n0) {
              ok = wait_p(0, j, 0x204);
              if (!ok) break;
              if (j == 0 && n > 0) {  // the epilogue of the previous item has read O0
                ok = mbar_wait_all(bar_o_free(0), (n - 1) & 1, abort_flag, 0x208);
                if (!ok) break;
              }
              FA2_TRACE_AT(trace_cta && n == 0, 16, j);
              tc_fence_after();
              issue_pv(0, j, g, j > 0);
              FA2_TRACE_AT(trace_cta && n == 0, 32, j);
              if (j + 1 == n0) umma_commit_w(bar_o_done(0));
              if (j + 1 < n1) {
                ok = wait_kv(g + 1);
                if (!ok) break;
                FA2_TRACE_AT(trace_cta && n == 0, 33, j);
                issue_s(1, j + 1, g + 1);  // into the buffer PV0_j has just read
                if (j + 2 == n1) umma_commit_w(bar_q_empty);  // the item's last S
              }
              FA2_TRACE_AT(trace_cta && n == 0, 17, j);
            }
            ok = wait_p(1, j, 0x205);
            if (!ok) break;
            if (j == 0 && n > 0) {
              ok = mbar_wait_all(bar_o_free(1), (n - 1) & 1, abort_flag, 0x209);
              if (!ok) break;
            }
            FA2_TRACE_AT(trace_cta && n == 0, 18, j);
            tc_fence_after();
            issue_pv(1, j, g, j > 0);
            FA2_TRACE_AT(trace_cta && n == 0, 35, j);
            umma_commit_w(bar_kv_empty(g % C::STAGES));  // K and V of this key tile fully consumed
            if (j + 1 == n1) umma_commit_w(bar_o_done(1));
            if (j + 2 < n0) {
              ok = wait_kv(g + 2);
              if (!ok) break;
              FA2_TRACE_AT(trace_cta && n == 0, 36, j);
              issue_s(0, j + 2, g + 2);  // into the buffer PV1_j has just read
            }
            FA2_TRACE_AT(trace_cta && n == 0, 19, j);
          }
        } else {
          for (int j = 0; j < n1 && ok; ++j) {
            const int g = kg + j;
            if (j < n0) {
              ok = wait_p(0, j, 0x204);
              if (!ok) break;
              if (j == 0 && n > 0) {  // the epilogue of the previous item has read O0
                ok = mbar_wait_all(bar_o_free(0), (n - 1) & 1, abort_flag, 0x208);
                if (!ok) break;
              }
              FA2_TRACE_AT(trace_cta && n == 0, 16, j);
              tc_fence_after();
              issue_pv(0, j, g, j > 0);
              if (j + 1 < n0) {
                ok = wait_kv(g + 1);
                if (!ok) break;
                issue_s(0, j + 1, g + 1);  // overwrites S0/P0 after PV0 in issue order
                FA2_TRACE_AT(trace_cta && n == 0, 17, j);
              } else {
                umma_commit_w(bar_o_done(0));
              }
            }
            if (EARLY && j + 1 == n1 && n0 == n1) {
              // Tile 0 is done with this item. While tile 1 forms its
              // last P, the next item's Q and first K/V tile may arrive: if they
              // do first, issue the next item's S0 of its first key tile now, so
              // that tile 0 (after its epilogue) starts the next item instead of
              // waiting for this item's last PV1; if P1 comes first, PV1 goes
              // first as before. Every S of this item is already issued (q_empty),
              // and the K/V slot of key tile kg + n1 is not this item's last
              // (STAGES >= 2). The poll is bounded like every other wait.
              // Items whose tile 1 has one key tile more (causal) keep the
              // plain order: there the early start measured 1-9 % slower, since
              // it shifts the two tiles' phases against each other.
              next_item = take_item_w(n + 1, 0x20A);
              if (next_item >= 0) {
                const int gp = jt1 + j;
                const int gk = kg + n1;
                const unsigned long long t_start = globaltimer();
                while (true) {
                  if (__all_sync(0xffffffffu, mbar_try_wait(bar_p_full(1, sp_k(gp)), sp_par(gp)))) break;
                  const bool kv_in = gk <= kv_waited ||
                                     mbar_try_wait(bar_kv_full(gk % C::STAGES), (gk / C::STAGES) & 1);
                  if (__all_sync(0xffffffffu, kv_in && mbar_try_wait(bar_q_full, (n + 1) & 1))) {
                    kv_waited = gk > kv_waited ? gk : kv_waited;
                    tc_fence_after();
                    issue_s(0, n0, kg + n1);  // phase index jt0 + n0: the next item's first
                    s0_early = true;
                    break;
                  }
                  if (*abort_flag) {
                    ok = false;
                    break;
                  }
                  if (globaltimer() - t_start > kWaitLimitNs) {
                    *abort_flag = 1;
                    report_timeout(0x20B);
                    ok = false;
                    break;
                  }
                }
                if (!ok) break;
              }
            }
            ok = wait_p(1, j, 0x205);
            if (!ok) break;
            if (j == 0 && n > 0) {
              ok = mbar_wait_all(bar_o_free(1), (n - 1) & 1, abort_flag, 0x209);
              if (!ok) break;
            }
            FA2_TRACE_AT(trace_cta && n == 0, 18, j);
            tc_fence_after();
            issue_pv(1, j, g, j > 0);
            umma_commit_w(bar_kv_empty(g % C::STAGES));  // K and V of this key tile fully consumed
            if (j + 1 < n1) {
              ok = wait_kv(g + 1);
              if (!ok) break;
              issue_s(1, j + 1, g + 1);
              if (j + 2 == n1) umma_commit_w(bar_q_empty);  // the item's last S: Q no longer read
              FA2_TRACE_AT(trace_cta && n == 0, 19, j);
            } else {
              umma_commit_w(bar_o_done(1));
            }
          }
        }
        kg += n1;
        jt0 += n0;
        jt1 += n1;
      }
      // drain: every UMMA of this CTA has finished before TMEM is released
      umma_commit_w(bar_drain);
      mbar_drain_wait(bar_drain, 0, 0x206);
    }
  } else {
    // ---------------------------------------------------------- softmax warps
    const int t = warp >> 3;              // query tile of this warpgroup
    const int h = (warp >> 2) & 1;        // key half: keys [64h, 64h+64) of each tile
    const int row = threadIdx.x & 127;    // TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    // this half's scores of the item's j-th key tile
    auto scol_of = [&](int j) -> uint32_t {
      if constexpr (C::ROT) return static_cast<uint32_t>((2 * j + t) % 3) * 128u + 64 * h;
      return (t ? C::COL_S1 : C::COL_S0) + 64 * h;
    };
    constexpr int DH = D / 2;                                    // O columns per half
    const uint32_t ocol = (t ? C::COL_O1 : C::COL_O0) + DH * h;
    float* xmax = reinterpret_cast<float*>(smem + C::OFF_XMAX) + t * 512 + row;  // + slot*256 + half*128
    float* xsum = reinterpret_cast<float*>(smem + C::OFF_XSUM) + t * 512 + row;  // + half*256 + which*128
    const float c = p.scale_log2;
    bool ok = true;
    int jt = 0;  // key tiles of this query tile over the CTA's items so far
    for (int n = 0; ok; ++n) {
      const int item = take_item(n, 0x306);
      if (item < 0) break;
      int pair, bh, n0, n1;
      fwd_decode_item(item, p.n_pairs, p.BH, p.head_group, p.causal != 0, pair, bh);
      tiles_of(pair, n0, n1);
      const int qt = 2 * pair + t;
      const int n_t = t ? n1 : n0;
      const int qrow = qt * C::BM + row;
      float m = -INFINITY;  // reference max of c * s, base-2 units (same in both halves)
      float l = 0.f;        // this half's row sum of the weights 2^(c s - m)
      float lr = 0.f;       // the same sum over the weights rounded to bf16
#ifdef FA2_TRACE
      const bool trace_row = trace_cta && n == 0 && row == 0 && h == 0;
      const bool trace_item = trace_cta && row == 0 && h == 0;
      const bool trace_last = trace_cta && n == 0 && row == 96 && h == 1;  // last warp of the tile
#endif
      FA2_TRACE_AT(trace_item, 24 + 4 * t, n);
      for (int j = 0; j < n_t; ++j) {
        const int jj = jt + j;
        FA2_TRACE_AT(trace_row, 8 * t + 0, j);
        ok = mbar_wait(bar_s_full(t, sp_k(jj)), sp_par(jj), abort_flag, 0x301);
        if (!ok) break;
        FA2_TRACE_AT(trace_row, 8 * t + 1, j);
        FA2_TRACE_AT(trace_last, 8 * t + 5, j);
        FA2_TRACE_AT(trace_cta && n == 0 && t == 0 && (threadIdx.x & 31) == 0, 56 + warp, j);
        FA2_TRACE_AT(trace_item && j == 0, 25 + 4 * t, n);
        tc_fence_after();
        const int k0 = j * C::BN + 64 * h;  // first key of this half
        // some row of the tile has keys of this tile masked (causal limit or Nk)
        const bool need_mask = (p.causal && j * C::BN + C::BN > qt * C::BM + 1 + p.kq_offset) ||
                               (j * C::BN + C::BN > p.Nk);
        const int lim = p.causal ? min(qrow + 1 + p.kq_offset, p.Nk) : p.Nk;  // keys [0, lim) allowed
        const uint32_t scol = scol_of(j);
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
        const int slot = jj & 1;
        xmax[slot * 256 + h * 128] = mx;
        mbar_arrive(bar_xmax(t, slot));
        ok = mbar_wait(bar_xmax(t, slot), (jj >> 1) & 1, abort_flag, 0x304);
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
        unsigned long long rs2 = f2(0.f, 0.f);
        float rr_lo = 0.f, rr_hi = 0.f;
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
              add_bf16x2(rr_lo, rr_hi, w);
            }
          } else {
            // masked keys get exponent -inf, hence weight exactly 0 (also when
            // c == 0, where the masked score -inf times c is NaN)
            const int nvalid = lim - k0;  // keys [k0, k0 + nvalid) of this half allowed
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int e = 32 * q + 2 * i;
              float x0, x1;
              f2_split(f2_fma(f2(s[e], s[e + 1]), c2, negm2), x0, x1);
              const float p0 = ex2(e < nvalid ? x0 : -INFINITY);
              const float p1 = ex2(e + 1 < nvalid ? x1 : -INFINITY);
              const uint32_t w = pack_bf16(p0, p1);
              pk[i] = w;
              rs2 = f2_add(rs2, f2(p0, p1));
              add_bf16x2(rr_lo, rr_hi, w);
            }
          }
          // P of keys [32q, 32q+32) of this half -> columns [16q, 16q+16): the scores
          // there are already in registers
          tmem_st16(lane_base + scol + 16 * q, pk);
        }
        FA2_TRACE_AT(trace_row, 8 * t + 3, j);
        FA2_TRACE_AT(trace_last, 8 * t + 6, j);
        float rs_lo, rs_hi;
        f2_split(rs2, rs_lo, rs_hi);
        l = l * alpha + (rs_lo + rs_hi);
        lr = lr * alpha + (rr_lo + rr_hi);
        // O must hold PV_0..PV_{j-1} complete. d = 128: it does, since S_j was
        // issued after them. d = 64 (S runs ahead): wait for PV_{j-1} first.
        // Each half rescales its own D/2 columns of O.
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
          if constexpr (C::ROT) {
            ok = mbar_wait(bar_pv_done(t), static_cast<uint32_t>((jj - 1) & 1), abort_flag, 0x307);
            if (!ok) break;
            tc_fence_after();
          }
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
        mbar_arrive(bar_p_full(t, sp_k(jj)));
        FA2_TRACE_AT(trace_row, 8 * t + 4, j);
        FA2_TRACE_AT(trace_last, 8 * t + 7, j);
        FA2_TRACE_AT(trace_cta && n == 0 && (threadIdx.x & 31) == 0, 40 + warp, j);
      }
      if (!ok) break;
      jt += n_t;
      // epilogue: O / l. The row sums over both halves are exchanged while the
      // item's last PV of this tile may still run.
      xsum[h * 256] = l;
      xsum[h * 256 + 128] = lr;
      mbar_arrive(bar_xsum(t));
      ok = mbar_wait(bar_xsum(t), n & 1, abort_flag, 0x305);
      if (!ok) break;
      l += xsum[(1 - h) * 256];
      lr += xsum[(1 - h) * 256 + 128];
      const float inv_l = 1.f / lr;
      ok = mbar_wait(bar_o_done(t), n & 1, abort_flag, 0x303);
      if (!ok) break;
      FA2_TRACE_AT(trace_item, 26 + 4 * t, n);
      tc_fence_after();
      // this half's D/2 columns, normalised and rounded to bf16 chunk by chunk
      uint4 w[DH / 8];
      uint32_t* wu = reinterpret_cast<uint32_t*>(w);
#pragma unroll
      for (int q = 0; q < DH / 32; ++q) {
        float part[32];
        tmem_ld32(lane_base + ocol + 32 * q, part);
#pragma unroll
        for (int i = 0; i < 16; ++i) wu[16 * q + i] = pack_bf16(part[2 * i] * inv_l, part[2 * i + 1] * inv_l);
      }
      // O has been read: the next item's first PV may overwrite it
      tc_fence_before();
      mbar_arrive(bar_o_free(t));
      {
        const int row0 = qt * C::BM + (warp & 3) * 32;  // query row of lane 0
        char* base = reinterpret_cast<char*>(p.o + (static_cast<size_t>(bh) * p.Nq + row0) * D + DH * h);
        store_rows_coalesced<DH / 8>(base, static_cast<size_t>(D) * 2, w, __ballot_sync(0xffffffffu, qrow < p.Nq));
      }
      if (qrow < p.Nq && h == 0)
        p.lse[static_cast<size_t>(bh) * p.Nq + qrow] = (m + __log2f(l)) * 0.69314718055994530942f;
      FA2_TRACE_AT(trace_item, 27 + 4 * t, n);
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::WARP_MMA) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace fa2
