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
//      and the main kernel's work-item counter zeroed. HBM-bound.
//   2. fa2_bwd_kernel: persistent, parallel over (128-key block, batch*head)
//      items; dK and dV accumulate in tensor memory over all query blocks, dQ
//      is added into an fp32 accumulator with reductions (layout below).
//   3. fa2_bwd_dq_convert: dQ = bf16(scale * accumulator).
#pragma once

#include <type_traits>

#include "exp2_poly.cuh"
#include "sm100_ptx.cuh"

namespace fa2 {


// ------------------------------------------------------------- preprocess (B1)
struct BwdPreParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;
  float* dq_acc;   // [BH][Np][d]
  float* delta;    // [BH][Np]: -D (negated, so the kernels add it)
  float* lse2;     // [BH][Np]: -LSE * log2 e (negated likewise)
  unsigned int* counter;  // work-item counter of the main kernel
  int N;
  int Np;
};

// Grid (row blocks, batch*head). 16 threads per row (d = 128) or 8 (d = 64),
// 16 bytes of O and dO per thread.
template <int D>
__global__ void __launch_bounds__(256) fa2_bwd_pre_kernel(const BwdPreParams p) {
  constexpr int TPR = D / 8;            // threads per row
  constexpr int RPB = 256 / TPR;        // rows per block per sweep
  const int sub = threadIdx.x % TPR;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *p.counter = 0u;
  const long long bh = blockIdx.y;
  for (int n = blockIdx.x * RPB + threadIdx.x / TPR; n < p.Np; n += gridDim.x * RPB) {
    const long long r = bh * p.Np + n;  // row of the [BH][Np] workspace arrays
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
      p.delta[r] = -acc;
      p.lse2[r] = (n < p.N) ? p.lse[static_cast<size_t>(bh) * p.N + n] * -1.4426950408889634f
                            : -INFINITY;
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
  int head8;            // N * d / 8: groups of 8 elements per head
  float scale;
};

// Grid (element blocks, batch*head). Within a head the accumulator and dQ are
// both row-major with row stride d (the accumulator's padding rows come last),
// so element e of the head is at offset e in both.
__global__ void __launch_bounds__(256) fa2_bwd_dq_convert_kernel(const BwdConvertParams p) {
  const size_t bh = blockIdx.y;
  const float* src_head = p.dq_acc + bh * p.Np * p.d;
  __nv_bfloat16* dst_head = p.dq + bh * p.N * p.d;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < p.head8; t += gridDim.x * blockDim.x) {
    const float4* src = reinterpret_cast<const float4*>(src_head + static_cast<size_t>(t) * 8);
    const float4 a = src[0];
    const float4 b = src[1];
    uint4 w;
    w.x = pack_bf16(a.x * p.scale, a.y * p.scale);
    w.y = pack_bf16(a.z * p.scale, a.w * p.scale);
    w.z = pack_bf16(b.x * p.scale, b.y * p.scale);
    w.w = pack_bf16(b.z * p.scale, b.w * p.scale);
    *reinterpret_cast<uint4*>(dst_head + static_cast<size_t>(t) * 8) = w;
  }
}


// ------------------------------------------------------------ main kernel (B2)
// Persistent: one CTA per SM takes work items (128-key block j, batch*head)
// from a counter in the workspace, longest first within groups of heads
// (causal: low j sees the most query blocks). Per item, query blocks i stream
// through a two-stage TMA ring (causal: only the blocks that see block j, the
// diagonal one first; with Nq != Nk query i sees keys <= i + Nk - Nq).
//   warp 16       TMA producer and scheduler: fetches the next item, hands it to
//                 the other warps through a two-slot ring, loads K_j, V_j once the
//                 previous item's MMAs are done, then Q_i with LSE2_i and D_i (two
//                 stages) and dO_i (one buffer at d = 128, two at d = 64)
//   (warps 16 and 17 run converged: the whole warp executes the loop and
//   elect.sync inside each copy / MMA instruction picks the issuing lane)
//   warp 17       MMA issuer + TMEM owner, per step, in this order:
//                   S^T = K Q_i^T,  dP^T = V dO_i^T          (keys on TMEM lanes)
//                   dV += P^T dO_i    (P^T from TMEM)
//                   dK += dS^T Q_i    (dS^T from smem, K-major)
//                   d = 128: dQ^T = K^T dS^T (d on lanes; dS^T read MN-major)
//                   d =  64: dQ   = dS K     (queries on lanes)
//   warp 18       reductions and stores: adds each step's staged dQ tile into
//                 the fp32 accumulator with TMA tensor reductions and, after an
//                 item, writes its dK and dV with TMA tensor stores
//   warps 0-15    four elementwise warpgroups; warpgroup g owns query columns
//                 [32g, 32g + 32) of a step and thread r key row r. P^T =
//                 exp2(c S^T - LSE2) goes back into TMEM over the group's own
//                 S^T columns; dS^T = P^T (dP^T - D) goes to swizzled smem; then
//                 the group's share of dQ goes to the fp32 accumulator: at
//                 d = 128 rows d < 64 through the staging buffer and warp 18,
//                 the rest with red.global; at d = 64 all through the staging
//                 buffer. No row statistics are needed (P comes from the saved
//                 LSE), so the groups never exchange data. After an item's last
//                 step they stage dV and scale * dK for warp 18's stores, while
//                 the MMA warp already starts the next item.
// Tensor memory: S^T [0,128) (P^T of group g in [32g, 32g+16)), dP^T [128,256),
// dV [256,256+D), dK [256+D,256+2D); dQ^T (d = 128) reuses the dP^T columns once
// dS is in smem, dQ (d = 64) has [384,448).
// Every barrier phase is counted over the whole sequence of items: `gs` counts
// steps, `n` counts items.
template <int D>
struct BwdCfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int BM = 128;                      // query rows per step
  static constexpr int BN = 128;                      // keys per item
  static constexpr int STAGES = 2;                    // Q (with LSE2 and D) stages
  // dO stages: dO_i is last read by dV_i in the middle of step i, half a step
  // before dP of step i+1 needs the next tile, so d = 128 single-buffers it and
  // spends the 32 KB on the dQ staging buffer
  static constexpr int DO_STAGES = (D == 128) ? 1 : 2;
  static constexpr int CHUNKS = D / 64;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int VEC_BYTES = 512;               // 128 fp32
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE_BYTES;
  static constexpr int OFF_Q = 2 * TILE_BYTES;                    // + s * TILE_BYTES
  static constexpr int OFF_DO = OFF_Q + STAGES * TILE_BYTES;      // + s * TILE_BYTES
  static constexpr int OFF_DS = OFF_DO + DO_STAGES * TILE_BYTES;  // 128 x 128 bf16
  // dQ staging for the TMA reductions: two 128-byte-swizzled boxes of
  // [128 query rows][32 fp32], i.e. d columns [0, 64) of one step's dQ tile
  static constexpr int OFF_STG = OFF_DS + 32768;
  static constexpr int STG_BOX_BYTES = 16384;
  static constexpr int OFF_VEC = OFF_STG + 2 * STG_BOX_BYTES;     // [s][LSE2 | D]
  static constexpr int OFF_BAR = OFF_VEC + STAGES * 2 * VEC_BYTES;
  // kv_full, kv_empty, st_full[S], st_empty[S], s_full, dp_full, p_ready,
  // ds_ready, dsm_free, dq_full, dq_empty, dkv_done, dkv_free, drain,
  // item_full[2], item_empty[2], do_full[DS], do_empty[DS], staged, stg_free,
  // epi_staged, dsbuf_free, epi_go
  static constexpr int NUM_BARS = 2 + 2 * STAGES + 10 + 4 + 2 * DO_STAGES + 5;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;         // tmem slot, abort, items[2]
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  // d = 128 uses 231,6xx bytes: there is no room for alignment slack, so the
  // kernel checks that the dynamic shared memory base is 1024-byte aligned
  static constexpr bool NEEDS_ALIGNED_BASE = SMEM_BYTES + 1024 > 232448;
  static constexpr int SMEM_ALLOC = NEEDS_ALIGNED_BASE ? SMEM_BYTES : SMEM_BYTES + 1024;
  static constexpr int NWG = 4;                       // elementwise warpgroups
  static constexpr int CW = 128 / NWG;                 // query columns per group
  static constexpr int WARP_TMA = 4 * NWG, WARP_MMA = 4 * NWG + 1, WARP_RED = 4 * NWG + 2;
  static constexpr int THREADS = 32 * (4 * NWG + 3);
  // groups of 4 exponentials (of CW / 4 per thread and step) that P^T takes on
  // the FMA pipe instead of MUFU: d = 128, 2 of 8 (measured +1-1.6 % over 0, 1
  // and 3); d = 64, none (measured 1-3 % faster than 1, 2 or 3)
  static constexpr int POLY_GROUPS = (D == 128) ? 2 : 0;
  static constexpr int ELEM_THREADS = 128 * NWG;
  // threads that stage dQ for the TMA reductions: d = 128, the warps whose
  // TMEM lanes (d rows of dQ^T) are [0, 64); d = 64, all (each group its own
  // 16 d columns). The other d = 128 warps reduce their rows with red.global.
  static constexpr int STG_THREADS = (D == 128) ? ELEM_THREADS / 2 : ELEM_THREADS;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
  // dQ layout: d = 128 computes dQ^T (d on lanes), so each warp reduction adds
  // 128 contiguous bytes of one query row: measured faster than 16-byte vector
  // reductions over scattered rows, which the L2 handles per half-filled sector.
  // d = 64 cannot (M would be 64) and uses dQ with queries on lanes.
  static constexpr bool DQ_T = (D == 128);
  // d = 128 has no free columns left: dQ reuses the dP^T columns once dS is in smem
  static constexpr bool DQ_IN_DP = (D == 128);
  static constexpr uint32_t COL_DQ = DQ_IN_DP ? COL_DP : 256 + 2 * D;
};

struct BwdParams {
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dq_acc;          // [BH][Np][d]
  const float* lse2;      // [BH][Np]
  const float* delta;     // [BH][Np]
  unsigned int* counter;  // next work item (zeroed by the preprocess kernel)
  int Np;                 // query rows rounded up to 128
  int BH;
  int n_ktiles;           // key tiles: ceil(Nk / 128)
  int n_qtiles;           // query tiles: Np / 128
  int kq_offset;          // Nk - Nq: causal query i sees keys j <= i + kq_offset
  int causal;
  int head_group;         // heads per causal scheduling group (see decode_item)
  float scale;
  float scale_log2;
};

// One float from shared memory. Used for the per-column LSE and D values, whose
// address is the same in every lane of a warp: as 32-bit loads those broadcasts
// cost one wavefront each, while the 128-bit vector loads the compiler would
// otherwise merge them into measured ~6.5 wavefronts each (ncu) -- shared
// memory bandwidth the tensor core's operand reads compete for.
__device__ __forceinline__ float lds_f32(const float* ptr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(ptr))));
  return v;
}

__device__ __forceinline__ void red_add(float* addr, float a) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(a) : "memory");
}

// Byte offset of 16-byte unit u (0..15) of row r in a [128][128] bf16 tile
// stored as two K-major 128-byte-swizzled halves of 64 columns.
__device__ __forceinline__ uint32_t sw128_offset(int r, int u) {
  return static_cast<uint32_t>((u >> 3) * 16384 + r * 128 + (((u & 7) ^ (r & 7)) << 4));
}

// Work item -> (key tile, batch*head). Non-causal items all cost the same: the
// key tiles of one head are consecutive, so they run together and share the
// head's Q/dO in L2. Causal items come in groups of head_group heads (their Q/dO
// stay in L2 while the group runs); inside a group the key tile is the slow
// index, so the items with the most query blocks come first.
__device__ __forceinline__ void decode_item(int item, int n_ktiles, int BH, int head_group,
                                            bool causal, int& ktile, int& bh) {
  if (!causal) {
    bh = item / n_ktiles;
    ktile = item - bh * n_ktiles;
    return;
  }
  const int group_items = head_group * n_ktiles;
  const int grp = item / group_items;
  const int r = item - grp * group_items;
  const int heads = min(head_group, BH - grp * head_group);
  ktile = r / heads;
  bh = grp * head_group + (r - ktile * heads);
}

// WITH_DQ = false is the dK/dV-only variant used when dQ comes from the
// separate query-parallel kernel (fa2_bwd_dq_kernel). tm_dq maps the fp32 dQ
// accumulator for the TMA reductions, tm_dk / tm_dv the bf16 outputs for the
// TMA stores of the epilogue.
template <int D, bool WITH_DQ>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    fa2_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dk,
                   const __grid_constant__ CUtensorMap tm_dv, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (C::NEEDS_ALIGNED_BASE && (smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) report_timeout(0x1000);  // layout assumption broken: refuse to run
    return;
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = p.n_ktiles * p.BH;
#ifdef FA2_TRACE
  const bool trace_cta = blockIdx.x == 7;
#endif

  const uint32_t bar_kv_full = sbase + C::OFF_BAR;
  const uint32_t bar_kv_empty = bar_kv_full + 8;
  auto bar_st_full = [&](int s) { return sbase + C::OFF_BAR + 8 * (2 + s); };
  auto bar_st_empty = [&](int s) { return sbase + C::OFF_BAR + 8 * (2 + C::STAGES + s); };
  const uint32_t bar_s_full = sbase + C::OFF_BAR + 8 * (2 + 2 * C::STAGES);
  const uint32_t bar_dp_full = bar_s_full + 8;
  const uint32_t bar_p_ready = bar_s_full + 16;
  const uint32_t bar_ds_ready = bar_s_full + 24;
  const uint32_t bar_dsm_free = bar_s_full + 32;
  const uint32_t bar_dq_full = bar_s_full + 40;
  const uint32_t bar_dq_empty = bar_s_full + 48;
  const uint32_t bar_dkv_done = bar_s_full + 56;
  const uint32_t bar_dkv_free = bar_s_full + 64;
  const uint32_t bar_drain = bar_s_full + 72;
  auto bar_item_full = [&](int q) { return bar_s_full + 80 + 8 * q; };
  auto bar_item_empty = [&](int q) { return bar_s_full + 96 + 8 * q; };
  auto bar_do_full = [&](int s) { return bar_s_full + 112 + 8 * s; };
  auto bar_do_empty = [&](int s) { return bar_s_full + 112 + 8 * (C::DO_STAGES + s); };
  const uint32_t bar_staged = bar_s_full + 112 + 16 * C::DO_STAGES;
  const uint32_t bar_stg_free = bar_staged + 8;
  const uint32_t bar_epi_staged = bar_staged + 16;
  const uint32_t bar_dsbuf_free = bar_staged + 24;
  const uint32_t bar_epi_go = bar_staged + 32;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);  // [2]

  FA2_TRACE_AT(trace_cta && threadIdx.x == 0, 30, 0);
  if (threadIdx.x == 0) {
    mbar_init(bar_kv_full, 1);
    mbar_init(bar_kv_empty, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_st_full(s), 1);
      mbar_init(bar_st_empty(s), 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_p_ready, C::ELEM_THREADS);
    mbar_init(bar_ds_ready, C::ELEM_THREADS);
    mbar_init(bar_dsm_free, 1);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dq_empty, C::ELEM_THREADS);
    mbar_init(bar_dkv_done, 1);
    mbar_init(bar_dkv_free, C::ELEM_THREADS);
    mbar_init(bar_drain, 1);
    for (int q = 0; q < 2; ++q) {
      mbar_init(bar_item_full(q), 1);
      // MMA thread + elementwise threads + reduction thread
      mbar_init(bar_item_empty(q), 2 + C::ELEM_THREADS);
    }
    for (int s = 0; s < C::DO_STAGES; ++s) {
      mbar_init(bar_do_full(s), 1);
      mbar_init(bar_do_empty(s), 1);
    }
    mbar_init(bar_staged, C::STG_THREADS);
    mbar_init(bar_stg_free, 1);
    mbar_init(bar_epi_staged, C::ELEM_THREADS);
    mbar_init(bar_dsbuf_free, 1);
    mbar_init(bar_epi_go, 1);
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
    prefetch_tensormap(&tm_do);
    prefetch_tensormap(&tm_dq);
    prefetch_tensormap(&tm_dk);
    prefetch_tensormap(&tm_dv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  FA2_TRACE_AT(trace_cta && threadIdx.x == 0, 31, 0);

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
  // causal: the first query tile that sees key tile ktile (query i sees keys
  // j <= i + kq_offset, the mask aligned to the bottom-right corner)
  auto qfirst = [&](int ktile) {
    const int x = ktile * C::BN - p.kq_offset;
    return p.causal && x > 0 ? x / C::BM : 0;
  };
  auto steps_of = [&](int ktile) { return p.n_qtiles - qfirst(ktile); };

  if (warp == C::WARP_TMA) {
    // --------------------------------------------------- scheduler + TMA producer
    // The whole warp runs this loop converged; elect.sync inside each copy and
    // expect_tx picks the issuing lane (see umma_ss2_w).
    {
      int last_st_parity[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) last_st_parity[s] = -1;
      int last_do_parity[C::DO_STAGES];
      for (int s = 0; s < C::DO_STAGES; ++s) last_do_parity[s] = -1;
      int last_kv_parity = -1;
      bool ok = true;
      int gs = 0;
      for (int n = 0; ok; ++n) {
        int item = 0;
        if (lane == 0) item = static_cast<int>(atomicAdd(p.counter, 1u));
        item = __shfl_sync(0xffffffffu, item, 0);
        if (item >= n_items) item = -1;
        if (n >= 2) ok = mbar_wait_all(bar_item_empty(n & 1), ((n >> 1) - 1) & 1, abort_flag, 0x1100);
        if (!ok) break;
        if (lane == 0) {
          item_slot[n & 1] = item;
          mbar_arrive(bar_item_full(n & 1));
        }
        __syncwarp();
        if (item < 0) break;
        int ktile, bh;
        decode_item(item, p.n_ktiles, p.BH, p.head_group, p.causal != 0, ktile, bh);
        const int i_first = qfirst(ktile);
        const int n_iter = steps_of(ktile);
        for (int it = 0; it < n_iter && ok; ++it, ++gs) {
          const int i = i_first + it;
          const int s = gs % C::STAGES;
          FA2_TRACE_AT(trace_cta && n == 0, 54, it);
          if (gs >= C::STAGES) ok = mbar_wait_all(bar_st_empty(s), ((gs / C::STAGES) - 1) & 1, abort_flag, 0x1101);
          if (!ok) break;
          FA2_TRACE_AT(trace_cta && n == 0, 52, it);
          if (it == 1 || n_iter == 1) {
            // K_j, V_j (after the first step's Q/dO is on its way) once the
            // previous item's MMAs are done with the buffers
            if (n >= 1) ok = mbar_wait_all(bar_kv_empty, (n - 1) & 1, abort_flag, 0x1104);
            if (!ok) break;
            mbar_arrive_expect_tx_w(bar_kv_full, 2 * C::TILE_BYTES);
            for (int c = 0; c < C::CHUNKS; ++c) {
              tma_load_3d_w(sbase + C::OFF_K + c * C::CHUNK_BYTES, &tm_k, bar_kv_full, c * 64, ktile * C::BN, bh);
              tma_load_3d_w(sbase + C::OFF_V + c * C::CHUNK_BYTES, &tm_v, bar_kv_full, c * 64, ktile * C::BN, bh);
            }
            last_kv_parity = n & 1;
          }
          const uint32_t bar = bar_st_full(s);
          mbar_arrive_expect_tx_w(bar, C::TILE_BYTES + 2 * C::VEC_BYTES);
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_3d_w(sbase + C::OFF_Q + s * C::TILE_BYTES + c * C::CHUNK_BYTES, &tm_q, bar,
                        c * 64, i * C::BM, bh);
          const size_t voff = static_cast<size_t>(bh) * p.Np + static_cast<size_t>(i) * C::BM;
          const uint32_t vec = sbase + C::OFF_VEC + s * 2 * C::VEC_BYTES;
          bulk_load_w(vec, p.lse2 + voff, C::VEC_BYTES, bar);
          bulk_load_w(vec + C::VEC_BYTES, p.delta + voff, C::VEC_BYTES, bar);
          FA2_TRACE_AT(trace_cta && n == 0, 53, it);
          last_st_parity[s] = (gs / C::STAGES) & 1;
          // dO_i once dV of the step that last used this dO buffer is done
          const int ds = gs % C::DO_STAGES;
          if (gs >= C::DO_STAGES)
            ok = mbar_wait_all(bar_do_empty(ds), ((gs / C::DO_STAGES) - 1) & 1, abort_flag, 0x1105);
          if (!ok) break;
          mbar_arrive_expect_tx_w(bar_do_full(ds), C::TILE_BYTES);
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_3d_w(sbase + C::OFF_DO + ds * C::TILE_BYTES + c * C::CHUNK_BYTES, &tm_do,
                        bar_do_full(ds), c * 64, i * C::BM, bh);
          last_do_parity[ds] = (gs / C::DO_STAGES) & 1;
        }
      }
      // never leave the CTA with copies still landing in its shared memory
      if (last_kv_parity >= 0) mbar_drain_wait(bar_kv_full, last_kv_parity, 0x1102);
      for (int s = 0; s < C::STAGES; ++s)
        if (last_st_parity[s] >= 0) mbar_drain_wait(bar_st_full(s), last_st_parity[s], 0x1103);
      for (int s = 0; s < C::DO_STAGES; ++s)
        if (last_do_parity[s] >= 0) mbar_drain_wait(bar_do_full(s), last_do_parity[s], 0x1106);
    }
  } else if (warp == C::WARP_MMA) {
    // --------------------------------------------------------------- MMA issuer
    // The whole warp runs this loop converged; elect.sync inside each MMA and
    // commit picks the issuing lane (see umma_ss2_w).
    {
      constexpr uint32_t IDESC_SS = idesc_bf16(128, 128, false, false);   // S^T, dP^T
      constexpr uint32_t IDESC_KV = idesc_bf16(128, D, false, true);      // dV, dK
      constexpr uint32_t IDESC_QT = idesc_bf16(128, 128, true, true);     // dQ^T (d = 128)
      constexpr uint32_t IDESC_Q = idesc_bf16(128, D, true, true);        // dQ (d = 64)
      // descriptor halves of every operand buffer, built once
      const SDesc dK = sdesc_make(sbase + C::OFF_K, 16, 1024);                // K-major
      const SDesc dV = sdesc_make(sbase + C::OFF_V, 16, 1024);
      const SDesc dQk = sdesc_make(sbase + C::OFF_Q, 16, 1024);
      const SDesc dOk = sdesc_make(sbase + C::OFF_DO, 16, 1024);
      const SDesc dQm = sdesc_make(sbase + C::OFF_Q, C::CHUNK_BYTES, 1024);   // MN-major
      const SDesc dOm = sdesc_make(sbase + C::OFF_DO, C::CHUNK_BYTES, 1024);
      const SDesc dKm = sdesc_make(sbase + C::OFF_K, C::CHUNK_BYTES, 1024);
      const SDesc dSk = sdesc_make(sbase + C::OFF_DS, 16, 1024);
      const SDesc dSm = sdesc_make(sbase + C::OFF_DS, C::CHUNK_BYTES, 1024);
      constexpr uint32_t TILE16 = C::TILE_BYTES / 16;  // stage stride in descriptor units
      auto kmaj = [](int k) -> uint32_t { return ((k >> 2) * C::CHUNK_BYTES + (k & 3) * 32) >> 4; };
      auto issue_s = [&](int g) {  // S^T = K Q_i^T for global step g
        const uint32_t qlo = dQk.lo + (g % C::STAGES) * TILE16;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          umma_ss2_w(tmem + C::COL_S, dK.lo + kmaj(k), dK.hi, qlo + kmaj(k), dQk.hi, IDESC_SS,
                   k > 0 ? 1u : 0u);
        umma_commit_w(bar_s_full);
      };
      bool ok = true;
      int gs = 0;
      for (int n = 0; ok; ++n) {
        const int item = take_item_w(n, 0x1209);
        if (item < 0) break;
        int ktile, bh;
        decode_item(item, p.n_ktiles, p.BH, p.head_group, p.causal != 0, ktile, bh);
        const int n_iter = steps_of(ktile);
        FA2_TRACE_AT(trace_cta, 40, n);
        ok = mbar_wait_all(bar_kv_full, n & 1, abort_flag, 0x1201) &&
             mbar_wait_all(bar_st_full(gs % C::STAGES), (gs / C::STAGES) & 1, abort_flag, 0x1202);
        if (!ok) break;
        FA2_TRACE_AT(trace_cta, 41, n);
        tc_fence_after();
        // S^T of the item's first step: the elementwise warps read the previous
        // S^T before its p_ready, and its P^T is read by a dV issued earlier
        issue_s(gs);
        for (int it = 0; it < n_iter && ok; ++it) {
          const int g = gs + it;
          const int s = g % C::STAGES;
          const uint32_t acc0 = it > 0 ? 1u : 0u;
          FA2_TRACE_AT(trace_cta && n == 0, 16, it);
          if (WITH_DQ && C::DQ_IN_DP && g > 0) {  // the dP^T columns hold dQ of step g-1 until read out
            ok = mbar_wait_all(bar_dq_empty, (g - 1) & 1, abort_flag, 0x1203);
            if (!ok) break;
            tc_fence_after();
          }
          FA2_TRACE_AT(trace_cta && n == 0, 17, it);
          const int ds = g % C::DO_STAGES;
          ok = mbar_wait_all(bar_do_full(ds), (g / C::DO_STAGES) & 1, abort_flag, 0x120B);
          if (!ok) break;
          tc_fence_after();
          const uint32_t dolo = dOk.lo + ds * TILE16;
#pragma unroll
          for (int k = 0; k < D / 16; ++k)  // dP^T = V dO_i^T
            umma_ss2_w(tmem + C::COL_DP, dV.lo + kmaj(k), dV.hi, dolo + kmaj(k), dOk.hi, IDESC_SS,
                     k > 0 ? 1u : 0u);
          umma_commit_w(bar_dp_full);
          // dV += P^T dO_i once every group has written P^T
          ok = mbar_wait_all(bar_p_ready, g & 1, abort_flag, 0x1204);
          if (!ok) break;
          if (it == 0 && n > 0) {  // the previous item's dK, dV have been read out
            ok = mbar_wait_all(bar_dkv_free, (n - 1) & 1, abort_flag, 0x120A);
            if (!ok) break;
          }
          FA2_TRACE_AT(trace_cta && n == 0, 18, it);
          tc_fence_after();
          const uint32_t domlo = dOm.lo + ds * TILE16;
#pragma unroll
          for (int k = 0; k < C::BM / 16; ++k) {
            // queries 16k..16k+15 sit in group g = 16k / CW at column CW g + (16k mod CW) / 2
            const uint32_t pcol = C::COL_S + C::CW * ((16 * k) / C::CW) + ((16 * k) % C::CW) / 2;
            umma_ts2_w(tmem + C::COL_DV, tmem + pcol, domlo + k * (2048 >> 4), dOm.hi, IDESC_KV,
                     k > 0 ? 1u : acc0);
          }
          umma_commit_w(bar_do_empty(ds));  // dV was the last reader of dO_i
          if (it + 1 < n_iter) {
            FA2_TRACE_AT(trace_cta && n == 0, 50, it);
            ok = mbar_wait_all(bar_st_full((g + 1) % C::STAGES), ((g + 1) / C::STAGES) & 1, abort_flag,
                           0x1208);
            if (!ok) break;
            FA2_TRACE_AT(trace_cta && n == 0, 51, it);
            tc_fence_after();
            issue_s(g + 1);
          }
          // dK += dS^T Q_i and dQ once dS^T is in smem
          ok = mbar_wait_all(bar_ds_ready, g & 1, abort_flag, 0x1205);
          if (!ok) break;
          FA2_TRACE_AT(trace_cta && n == 0, 19, it);
          tc_fence_after();
          auto issue_dk = [&]() {
            const uint32_t qmlo = dQm.lo + s * TILE16;
#pragma unroll
            for (int k = 0; k < C::BM / 16; ++k)
              umma_ss2_w(tmem + C::COL_DK, dSk.lo + kmaj(k), dSk.hi, qmlo + k * (2048 >> 4), dQm.hi,
                       IDESC_KV, k > 0 ? 1u : acc0);
          };
          // dK first: it is the last reader of Q_i, so the stage goes back to
          // the producer one GEMM earlier and the load of the query block two
          // steps ahead has that much longer to land (its TMA load takes
          // ~2000 cycles here). Measured at d = 128 against dQ first: +0.5-1.8 %
          // on four of five shapes; dK first without the early release: -1-5 %.
          issue_dk();
          umma_commit_w(bar_st_empty(s));  // Q_i (and its LSE2, D) no longer read
          if constexpr (WITH_DQ) {
            if (!C::DQ_IN_DP && g > 0) {  // dQ of step g-1 must be read out before it is overwritten
              ok = mbar_wait_all(bar_dq_empty, (g - 1) & 1, abort_flag, 0x1206);
              if (!ok) break;
              tc_fence_after();
            }
  #pragma unroll
            for (int k = 0; k < C::BN / 16; ++k) {  // reduction over the 128 keys
              if (C::DQ_T)  // dQ^T = K^T dS^T
                umma_ss2_w(tmem + C::COL_DQ, dKm.lo + k * (2048 >> 4), dKm.hi, dSm.lo + k * (2048 >> 4),
                         dSm.hi, IDESC_QT, k > 0 ? 1u : 0u);
              else  // dQ = dS K
                umma_ss2_w(tmem + C::COL_DQ, dSm.lo + k * (2048 >> 4), dSm.hi, dKm.lo + k * (2048 >> 4),
                         dKm.hi, IDESC_Q, k > 0 ? 1u : 0u);
            }
            umma_commit_w(bar_dq_full);
          }
          umma_commit_w(bar_dsm_free);
        }
        if (!ok) break;
        umma_commit_w(bar_dkv_done);  // dK, dV of this item complete
        umma_commit_w(bar_kv_empty);  // K_j, V_j no longer read
        gs += n_iter;
      }
      umma_commit_w(bar_drain);
      mbar_drain_wait(bar_drain, 0, 0x1207);
    }
  } else if (warp == C::WARP_RED) {
    // -------------------------------------------- dQ reductions, dK/dV stores
    // Step g's staged dQ tile (d columns [0, 64)) is added into the fp32
    // accumulator by TMA reductions; at the end of an item, dV (staged in the
    // dS^T buffer) and scale * dK (in the staging buffer) go out by TMA stores.
    // Each buffer is freed as soon as the TMA has read it. The staging buffer's
    // uses (one per step, then one per item) are counted in this same order by
    // the threads that stage dQ (stg_free); epi_go, one phase per item, tells
    // every elementwise thread that the item's dQ tiles have been read.
    if (lane == 0) {
      bool ok = true;
      int gs = 0;
      for (int n = 0; ok; ++n) {
        const int item = take_item(n, 0x1709);
        if (item < 0) break;
        int ktile, bh;
        decode_item(item, p.n_ktiles, p.BH, p.head_group, p.causal != 0, ktile, bh);
        const int i_first = qfirst(ktile);
        const int n_iter = steps_of(ktile);
        for (int it = 0; WITH_DQ && it < n_iter; ++it) {
          const int g = gs + it;
          ok = mbar_wait(bar_staged, g & 1, abort_flag, 0x1701);
          if (!ok) break;
          tma_reduce_add_3d(&tm_dq, sbase + C::OFF_STG, 0, (i_first + it) * C::BM, bh);
          tma_reduce_add_3d(&tm_dq, sbase + C::OFF_STG + C::STG_BOX_BYTES, 32, (i_first + it) * C::BM, bh);
          bulk_commit_group();
          bulk_wait_group_read0();
          mbar_arrive(bar_stg_free);
        }
        if (!ok) break;
        mbar_arrive(bar_epi_go);
        ok = mbar_wait(bar_epi_staged, n & 1, abort_flag, 0x1702);
        if (!ok) break;
        for (int c = 0; c < C::CHUNKS; ++c) {  // rows past N are not written by the TMA
          tma_store_3d(&tm_dv, sbase + C::OFF_DS + c * C::CHUNK_BYTES, c * 64, ktile * C::BN, bh);
          tma_store_3d(&tm_dk, sbase + C::OFF_STG + c * C::CHUNK_BYTES, c * 64, ktile * C::BN, bh);
        }
        bulk_commit_group();
        bulk_wait_group_read0();
        mbar_arrive(bar_dsbuf_free);
        mbar_arrive(bar_stg_free);
        gs += n_iter;
      }
      bulk_wait_group0();  // every reduction and store has landed before the kernel ends
    }
  } else {
    // ------------------------------------------------ elementwise groups (0-15)
    constexpr int CW = C::CW;
    const int g = warp >> 2;            // query-column group
    const int r = threadIdx.x & 127;    // TMEM lane: key row (S^T, dP^T, dK, dV)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float c = p.scale_log2;
    uint8_t* ds_base = smem + C::OFF_DS;
    bool ok = true;
    int gs = 0;
    for (int n = 0; ok; ++n) {
      const int item = take_item(n, 0x1309);
      if (item < 0) break;
      int ktile, bh;
      decode_item(item, p.n_ktiles, p.BH, p.head_group, p.causal != 0, ktile, bh);
      const int i_first = qfirst(ktile);
      const int n_iter = steps_of(ktile);
      FA2_TRACE_AT(trace_cta && threadIdx.x == 0, 44, n);
#ifdef FA2_TRACE
      // group 0: a thread of the first warp (dQ staging at d = 128); group 1: a
      // thread of the third warp (dQ reductions at d = 128)
      const bool trace_row = trace_cta && n == 0 && ((g == 0 && r == 0) || (g == 1 && r == 64));
#endif
      // dQ of step it (this group's share) -> fp32 accumulator: d columns [0, 64)
      // through the staging buffer and the TMA, the rest (d = 128) with
      // red.global. The TMEM columns are released as soon as the values are in
      // registers.
      const uint32_t stg = sbase + C::OFF_STG;
      // drain_ld: wait for dQ of step it, move this group's share into registers
      // and release the TMEM columns; drain_st: send the registers on.
      constexpr int DQW = C::DQ_T ? CW : D / C::NWG;
      float dqv[DQW];
      auto drain_ld = [&](int it) -> bool {
        if (!mbar_wait(bar_dq_full, (gs + it) & 1, abort_flag, 0x1304)) return false;
        FA2_TRACE_AT(trace_row, 8 * g + 4, it);
        tc_fence_after();
        if constexpr (C::DQ_T) {
          // lane r holds dQ^T[d = r][query CW g + q]
          tmem_ld32(lane_base + C::COL_DQ + CW * g, dqv);
        } else {
          // lane r holds dQ[query r][d]; this group stages d columns [16 g, 16 g + 16)
          static_assert(C::DQ_T || DQW == 16, "d = 64 stages all of dQ");
          tmem_ld16(lane_base + C::COL_DQ + DQW * g, dqv);
        }
        tc_fence_before();
        mbar_arrive(bar_dq_empty);
        FA2_TRACE_AT(trace_row, 60 + g, it);
        return true;
      };
      auto drain_st = [&](int it) -> bool {
        float* acc = p.dq_acc + (static_cast<size_t>(bh) * p.Np + static_cast<size_t>(i_first + it) * C::BM) * D;
        const int gg = gs + it;
        if constexpr (C::DQ_T) {
          if (r < 64) {
            // staged: row q of box r/32 holds query CW g + q; d = r sits in 16-byte
            // unit ((r mod 32) / 4) xor (row mod 8) of the 128-byte swizzle. This is
            // staging-buffer use gg + n: every earlier step and item epilogue used it.
            if (gg + n > 0 && !mbar_wait(bar_stg_free, (gg + n - 1) & 1, abort_flag, 0x1306)) return false;
            const uint32_t box = stg + (r >> 5) * C::STG_BOX_BYTES;
            const uint32_t unit = static_cast<uint32_t>((r & 31) >> 2);
            const uint32_t word = static_cast<uint32_t>(r & 3) * 4;
#pragma unroll
            for (int q = 0; q < CW; ++q) {
              const int row = CW * g + q;
              st_shared_f32(box + row * 128 + ((unit ^ (row & 7)) << 4) + word, dqv[q]);
            }
            FA2_TRACE_AT(trace_row, 62 + g, it);
            fence_async_smem();
            mbar_arrive(bar_staged);
          } else {
            // each warp instruction adds 32 consecutive d values of one query row
            float* col = acc + static_cast<size_t>(CW * g) * D + r;
#pragma unroll
            for (int q = 0; q < CW; ++q) red_add(col + static_cast<size_t>(q) * D, dqv[q]);
            FA2_TRACE_AT(trace_row, 62 + g, it);
          }
        } else {
          if (gg + n > 0 && !mbar_wait(bar_stg_free, (gg + n - 1) & 1, abort_flag, 0x1306)) return false;
#pragma unroll
          for (int u = 0; u < DQW / 4; ++u) {
            const int col = DQW * g + 4 * u;
            const uint32_t box = stg + (col >> 5) * C::STG_BOX_BYTES;
            const uint32_t unit = static_cast<uint32_t>((col & 31) >> 2);
            st_shared_v4(box + r * 128 + ((unit ^ (r & 7)) << 4), dqv[4 * u], dqv[4 * u + 1], dqv[4 * u + 2],
                         dqv[4 * u + 3]);
          }
          fence_async_smem();
          mbar_arrive(bar_staged);
        }
        FA2_TRACE_AT(trace_row, 8 * g + 5, it);
        return true;
      };
      auto drain = [&](int it) -> bool { return drain_ld(it) && drain_st(it); };
      for (int it = 0; it < n_iter; ++it) {
        const int i = i_first + it;
        const int gg = gs + it;
        const int s = gg % C::STAGES;
        // -LSE2 and -D of this step's query columns (stored negated, so they add)
        const float* nlse2 = reinterpret_cast<const float*>(smem + C::OFF_VEC + s * 2 * C::VEC_BYTES) + CW * g;
        const float* ndlt = nlse2 + 128;
        FA2_TRACE_AT(trace_row, 8 * g + 0, it);
        // LSE2 and D of this query block were written by the TMA (async proxy)
        ok = mbar_wait(bar_st_full(s), (gg / C::STAGES) & 1, abort_flag, 0x1300);
        if (!ok) break;
        FA2_TRACE_AT(trace_row, 48 + g, it);
        ok = mbar_wait(bar_s_full, gg & 1, abort_flag, 0x1301);
        if (!ok) break;
        FA2_TRACE_AT(trace_row, 8 * g + 1, it);
        FA2_TRACE_AT(trace_cta && threadIdx.x == 0 && it == 0, 43, n);
        tc_fence_after();
        // P^T for query columns [CW g, CW g + CW)
        uint32_t pk[CW / 2];
        {
          float sv[CW];
          tmem_ld32(lane_base + C::COL_S + CW * g, sv);
          FA2_TRACE_AT(trace_row, 56 + g, it);
          const unsigned long long c2 = f2(c, c);
          // keys past query q + off are masked; off >= 127 masks none
          const int off = i * C::BM + p.kq_offset - ktile * C::BN;
          const bool diag = p.causal && off < C::BN - 1;
          // the same loop twice, with and without the causal mask, so that the
          // common (unmasked) case has no branch between its independent groups
          auto form_p = [&](auto masked) {
#pragma unroll
            for (int e = 0; e < CW; e += 4) {
              const float4 l4 = make_float4(lds_f32(nlse2 + e), lds_f32(nlse2 + e + 1), lds_f32(nlse2 + e + 2),
                                            lds_f32(nlse2 + e + 3));
              float x0, x1, x2, x3;
              f2_split(f2_fma(f2(sv[e], sv[e + 1]), c2, f2(l4.x, l4.y)), x0, x1);
              f2_split(f2_fma(f2(sv[e + 2], sv[e + 3]), c2, f2(l4.z, l4.w)), x2, x3);
              float p0, p1, p2, p3;
              if (e / 4 < C::POLY_GROUPS) {  // FMA pipe: takes load off the MUFU unit
                exp2_poly2(x0, x1, p0, p1);
                exp2_poly2(x2, x3, p2, p3);
              } else {
                p0 = ex2(x0);
                p1 = ex2(x1);
                p2 = ex2(x2);
                p3 = ex2(x3);
              }
              if constexpr (decltype(masked)::value) {
                // query i*128 + q sees key ktile*128 + r only if r <= q + off
                const int q = CW * g + e;
                p0 = q + off < r ? 0.f : p0;
                p1 = q + 1 + off < r ? 0.f : p1;
                p2 = q + 2 + off < r ? 0.f : p2;
                p3 = q + 3 + off < r ? 0.f : p3;
              }
              pk[e / 2] = pack_bf16(p0, p1);
              pk[e / 2 + 1] = pack_bf16(p2, p3);
            }
          };
          if (diag)
            form_p(std::integral_constant<bool, true>());
          else
            form_p(std::integral_constant<bool, false>());
        }
        // P^T over the group's own first CW/2 S^T columns (already read above)
        FA2_TRACE_AT(trace_row, 58 + g, it);
        tmem_st16(lane_base + C::COL_S + CW * g, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_p_ready);
        FA2_TRACE_AT(trace_row, 8 * g + 2, it);
        // the previous step's dQ is ready by now (its MMAs ran while P^T was formed)
        if (WITH_DQ && it > 0) {
          ok = drain(it - 1);
          if (!ok) break;
        }
        // dS^T = P^T (dP^T - D) for the same columns, bf16 into the swizzled smem tile
        ok = mbar_wait(bar_dp_full, gg & 1, abort_flag, 0x1302);
        if (!ok) break;
        FA2_TRACE_AT(trace_row, 8 * g + 6, it);
        tc_fence_after();
        uint32_t dk[CW / 2];
        {
          float dp[CW];
          tmem_ld32(lane_base + C::COL_DP + CW * g, dp);
#pragma unroll
          for (int e = 0; e < CW; e += 4) {
            const float4 d4 = make_float4(lds_f32(ndlt + e), lds_f32(ndlt + e + 1), lds_f32(ndlt + e + 2),
                                          lds_f32(ndlt + e + 3));
            const unsigned long long pa = f2(__uint_as_float(pk[e / 2] << 16), __uint_as_float(pk[e / 2] & 0xFFFF0000u));
            const unsigned long long pb = f2(__uint_as_float(pk[e / 2 + 1] << 16), __uint_as_float(pk[e / 2 + 1] & 0xFFFF0000u));
            const unsigned long long da = f2_add(f2(dp[e], dp[e + 1]), f2(d4.x, d4.y));
            const unsigned long long db = f2_add(f2(dp[e + 2], dp[e + 3]), f2(d4.z, d4.w));
            float s0, s1, s2, s3;
            f2_split(f2_mul(pa, da), s0, s1);
            f2_split(f2_mul(pb, db), s2, s3);
            dk[e / 2] = pack_bf16(s0, s1);
            dk[e / 2 + 1] = pack_bf16(s2, s3);
          }
        }
        if (it == 0 && n > 0) {  // the TMA has read the previous item's dV staged there
          ok = mbar_wait(bar_dsbuf_free, (n - 1) & 1, abort_flag, 0x1307);
          if (!ok) break;
        } else if (gg > 0) {  // dK and dQ of the previous step have finished reading the dS^T tile
          ok = mbar_wait(bar_dsm_free, (gg - 1) & 1, abort_flag, 0x1303);
          if (!ok) break;
        }
        FA2_TRACE_AT(trace_row, 8 * g + 7, it);
#pragma unroll
        for (int u = 0; u < CW / 8; ++u) {
          const uint32_t off = sw128_offset(r, (CW / 8) * g + u);
          *reinterpret_cast<uint4*>(ds_base + off) = make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(bar_ds_ready);
        FA2_TRACE_AT(trace_row, 8 * g + 3, it);
      }
      if (WITH_DQ && ok) ok = drain(n_iter - 1);
      FA2_TRACE_AT(trace_cta && threadIdx.x == 0, 45, n);
      if (ok) ok = mbar_wait(bar_dkv_done, n & 1, abort_flag, 0x1305);
#ifdef FA2_TRACE
      FA2_TRACE_AT(trace_row, 32, 0);
      FA2_TRACE_AT(trace_cta && threadIdx.x == 0, 46, n);
#endif
      if (!ok) break;
      // epilogue: group g stages d columns [g D/4, (g+1) D/4) of dV (in the dS^T
      // buffer: the item's last dK and dQ MMAs are done) and of scale * dK (in the
      // staging buffer, once the TMA has read its last dQ tile), 128-byte-swizzled
      // like the tensor maps; the reduction warp stores them with the TMA. The
      // TMEM columns are released first.
      {
        constexpr int DW = D / C::NWG;
        tc_fence_after();
        float v[DW], w[DW];
        if constexpr (DW == 32) {
          tmem_ld32(lane_base + C::COL_DV + DW * g, v);
          tmem_ld32(lane_base + C::COL_DK + DW * g, w);
        } else {
          tmem_ld16(lane_base + C::COL_DV + DW * g, v);
          tmem_ld16(lane_base + C::COL_DK + DW * g, w);
        }
        tc_fence_before();
        mbar_arrive(bar_dkv_free);
        uint32_t pk[DW / 2];
#pragma unroll
        for (int e = 0; e < DW / 2; ++e) pk[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
#pragma unroll
        for (int u = 0; u < DW / 8; ++u) {
          const uint32_t off = sw128_offset(r, (DW / 8) * g + u);
          *reinterpret_cast<uint4*>(smem + C::OFF_DS + off) =
              make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
#pragma unroll
        for (int e = 0; e < DW / 2; ++e) pk[e] = pack_bf16(w[2 * e] * p.scale, w[2 * e + 1] * p.scale);
        // the TMA has read every dQ tile of this item from the staging buffer (and,
        // before those, the previous item's dK)
        ok = mbar_wait(bar_epi_go, n & 1, abort_flag, 0x1308);
        if (!ok) break;
#pragma unroll
        for (int u = 0; u < DW / 8; ++u) {
          const uint32_t off = sw128_offset(r, (DW / 8) * g + u);
          *reinterpret_cast<uint4*>(smem + C::OFF_STG + off) =
              make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
        fence_async_smem();
        mbar_arrive(bar_epi_staged);
      }
      FA2_TRACE_AT(trace_cta && threadIdx.x == 0, 47, n);
      gs += n_iter;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  FA2_TRACE_AT(trace_cta && threadIdx.x == 0, 33, 0);
  if (warp == C::WARP_MMA) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ------------------------------------------------------ dQ kernel (B3b)
// dQ by a separate, query-parallel kernel: one CTA per (128-row query block i,
// batch*head) loops over the key blocks j (causal: j <= i) and recomputes
//   S = Q_i K_j^T,  P = exp2(c S - LSE2),  dP = dO_i V_j^T,  dS = P (dP - D),
//   dQ_i += dS K_j   (accumulated in TMEM; scaled and stored once, no atomics).
// Queries sit on TMEM lanes, so LSE2 and D are one register per thread.
//   warp 16       TMA producer: Q_i, dO_i once, then K_j/V_j into a 2-stage ring
//   warp 17       MMA issuer: S_j, dP_j; after dS_j is in smem, S_{j+1}, dP_{j+1}
//                 and then dQ += dS_j K_j (so the next elementwise pass overlaps it)
//   warps 0-15    four elementwise warpgroups, group g owns keys [32g, 32g+32)
// Tensor memory: S [0,128), dP [128,256), dQ [256,256+D).
template <int D>
struct BwdDqCfg {
  static constexpr int BM = 128, BN = 128, STAGES = 2;
  static constexpr int CHUNKS = D / 64;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = TILE_BYTES;
  static constexpr int OFF_K = 2 * TILE_BYTES;                  // + s * 2 * TILE_BYTES
  static constexpr int OFF_V = 3 * TILE_BYTES;                  // + s * 2 * TILE_BYTES
  static constexpr int OFF_DS = TILE_BYTES * (2 + 2 * STAGES);  // 128 x 128 bf16, [query][key]
  static constexpr int OFF_BAR = OFF_DS + 32768;
  // q_full, kv_full[S], kv_empty[S], s_full, dp_full, ds_ready, dsm_free, dq_done, drain
  static constexpr int NUM_BARS = 1 + 2 * STAGES + 6;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NUM_BARS;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  static constexpr int NWG = 4, CW = 128 / NWG;
  static constexpr int WARP_TMA = 4 * NWG, WARP_MMA = 4 * NWG + 1;
  static constexpr int THREADS = 32 * (4 * NWG + 2);
  static constexpr int ELEM_THREADS = 128 * NWG;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DQ = 256;
  static constexpr int HEAD_GROUP = 16;
};

struct BwdDqParams {
  __nv_bfloat16* dq;
  const float* lse2;   // [BH][Np]
  const float* delta;  // [BH][Np]
  int N;
  int Np;
  int BH;
  int n_qtiles;
  int causal;
  float scale;
  float scale_log2;
};

template <int D>
__global__ void __launch_bounds__(BwdDqCfg<D>::THREADS, 1)
    fa2_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const BwdDqParams p) {
  using C = BwdDqCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Non-causal: grid (query tile, batch*head). Causal: 1-D grid in groups of
  // HEAD_GROUP heads with the query tiles that see the most key tiles first.
  int qtile, bh;
  if (!p.causal) {
    qtile = blockIdx.x;
    bh = blockIdx.y;
  } else {
    const int group_blocks = C::HEAD_GROUP * p.n_qtiles;
    const int grp = static_cast<int>(blockIdx.x) / group_blocks;
    const int r = static_cast<int>(blockIdx.x) - grp * group_blocks;
    const int heads = min(C::HEAD_GROUP, p.BH - grp * C::HEAD_GROUP);
    qtile = p.n_qtiles - 1 - r / heads;
    bh = grp * C::HEAD_GROUP + r % heads;
  }
  const int n_kv = p.causal ? qtile + 1 : p.n_qtiles;  // self-attention: key tiles = query tiles

  const uint32_t bar_q = sbase + C::OFF_BAR;
  auto bar_kv_full = [&](int s) { return sbase + C::OFF_BAR + 8 * (1 + s); };
  auto bar_kv_empty = [&](int s) { return sbase + C::OFF_BAR + 8 * (1 + C::STAGES + s); };
  const uint32_t bar_s_full = sbase + C::OFF_BAR + 8 * (1 + 2 * C::STAGES);
  const uint32_t bar_dp_full = bar_s_full + 8;
  const uint32_t bar_ds_ready = bar_s_full + 16;
  const uint32_t bar_dsm_free = bar_s_full + 24;
  const uint32_t bar_dq_done = bar_s_full + 32;
  const uint32_t bar_drain = bar_s_full + 40;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_kv_full(s), 1);
      mbar_init(bar_kv_empty(s), 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_ds_ready, C::ELEM_THREADS);
    mbar_init(bar_dsm_free, 1);
    mbar_init(bar_dq_done, 1);
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
    prefetch_tensormap(&tm_do);
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
        tma_load_3d(sbase + C::OFF_Q + c * C::CHUNK_BYTES, &tm_q, bar_q, c * 64, qtile * C::BM, bh);
        tma_load_3d(sbase + C::OFF_DO + c * C::CHUNK_BYTES, &tm_do, bar_q, c * 64, qtile * C::BM, bh);
      }
      int last_parity[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        const int s = j % C::STAGES;
        const int n = j / C::STAGES;
        if (n > 0) ok = mbar_wait(bar_kv_empty(s), (n - 1) & 1, abort_flag, 0x1401);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_kv_full(s), 2 * C::TILE_BYTES);
        for (int c = 0; c < C::CHUNKS; ++c) {
          tma_load_3d(sbase + C::OFF_K + s * 2 * C::TILE_BYTES + c * C::CHUNK_BYTES, &tm_k,
                      bar_kv_full(s), c * 64, j * C::BN, bh);
          tma_load_3d(sbase + C::OFF_V + s * 2 * C::TILE_BYTES + c * C::CHUNK_BYTES, &tm_v,
                      bar_kv_full(s), c * 64, j * C::BN, bh);
        }
        last_parity[s] = n & 1;
      }
      mbar_drain_wait(bar_q, 0, 0x1402);
      for (int s = 0; s < C::STAGES; ++s)
        if (last_parity[s] >= 0) mbar_drain_wait(bar_kv_full(s), last_parity[s], 0x1403);
    }
  } else if (warp == C::WARP_MMA) {
    // --------------------------------------------------------------- MMA issuer
    // The whole warp runs this loop converged; elect.sync inside each MMA and
    // commit picks the issuing lane (see umma_ss2_w).
    {
      constexpr uint32_t IDESC_SS = idesc_bf16(128, 128, false, false);  // S, dP
      constexpr uint32_t IDESC_DQ = idesc_bf16(128, D, false, true);     // dQ += dS K
      const SDesc dQk = sdesc_make(sbase + C::OFF_Q, 16, 1024);
      const SDesc dOk = sdesc_make(sbase + C::OFF_DO, 16, 1024);
      const SDesc dK = sdesc_make(sbase + C::OFF_K, 16, 1024);
      const SDesc dV = sdesc_make(sbase + C::OFF_V, 16, 1024);
      const SDesc dKm = sdesc_make(sbase + C::OFF_K, C::CHUNK_BYTES, 1024);
      const SDesc dSk = sdesc_make(sbase + C::OFF_DS, 16, 1024);
      constexpr uint32_t STAGE16 = 2 * C::TILE_BYTES / 16;
      auto kmaj = [](int k) -> uint32_t { return ((k >> 2) * C::CHUNK_BYTES + (k & 3) * 32) >> 4; };
      auto issue_s_dp = [&](int j) {  // S = Q K_j^T, dP = dO V_j^T
        const uint32_t klo = dK.lo + (j % C::STAGES) * STAGE16;
        const uint32_t vlo = dV.lo + (j % C::STAGES) * STAGE16;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          umma_ss2_w(tmem + C::COL_S, dQk.lo + kmaj(k), dQk.hi, klo + kmaj(k), dK.hi, IDESC_SS,
                   k > 0 ? 1u : 0u);
        umma_commit_w(bar_s_full);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          umma_ss2_w(tmem + C::COL_DP, dOk.lo + kmaj(k), dOk.hi, vlo + kmaj(k), dV.hi, IDESC_SS,
                   k > 0 ? 1u : 0u);
        umma_commit_w(bar_dp_full);
      };
      bool ok = mbar_wait_all(bar_q, 0, abort_flag, 0x1501) &&
                mbar_wait_all(bar_kv_full(0), 0, abort_flag, 0x1502);
      if (ok) {
        tc_fence_after();
        issue_s_dp(0);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        // the elementwise warps have read S_j and dP_j and written dS_j
        ok = mbar_wait_all(bar_ds_ready, j & 1, abort_flag, 0x1503);
        if (!ok) break;
        tc_fence_after();
        if (j + 1 < n_kv) {
          ok = mbar_wait_all(bar_kv_full((j + 1) % C::STAGES), ((j + 1) / C::STAGES) & 1, abort_flag, 0x1504);
          if (!ok) break;
          tc_fence_after();
          issue_s_dp(j + 1);
        }
        const uint32_t kmlo = dKm.lo + (j % C::STAGES) * STAGE16;
#pragma unroll
        for (int k = 0; k < C::BN / 16; ++k)  // dQ += dS_j K_j (reduction over keys)
          umma_ss2_w(tmem + C::COL_DQ, dSk.lo + kmaj(k), dSk.hi, kmlo + k * (2048 >> 4), dKm.hi,
                   IDESC_DQ, (j > 0 || k > 0) ? 1u : 0u);
        umma_commit_w(bar_dsm_free);
        umma_commit_w(bar_kv_empty(j % C::STAGES));
      }
      umma_commit_w(bar_dq_done);
      umma_commit_w(bar_drain);
      mbar_drain_wait(bar_drain, 0, 0x1505);
    }
  } else {
    // ------------------------------------------------ elementwise groups (0-15)
    constexpr int CW = C::CW;
    const int g = warp >> 2;           // key-column group
    const int r = threadIdx.x & 127;   // TMEM lane: query row
    const int qrow = qtile * C::BM + r;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const size_t vrow = static_cast<size_t>(bh) * p.Np + qrow;
    const float nlse2 = p.lse2[vrow];   // -LSE log2 e; -inf on padding rows: P = 0 there
    const float ndlt = p.delta[vrow];   // -D
    const unsigned long long c2 = f2(p.scale_log2, p.scale_log2);
    const unsigned long long nl2 = f2(nlse2, nlse2);
    const unsigned long long nd2 = f2(ndlt, ndlt);
    uint8_t* ds_base = smem + C::OFF_DS;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      ok = mbar_wait(bar_s_full, j & 1, abort_flag, 0x1601);
      if (!ok) break;
      tc_fence_after();
      const bool diag = p.causal && j == qtile;
      uint32_t pk[CW / 2];
      {
        float sv[CW];
        tmem_ld32(lane_base + C::COL_S + CW * g, sv);
#pragma unroll
        for (int e = 0; e < CW; e += 2) {
          float x0, x1;
          f2_split(f2_fma(f2(sv[e], sv[e + 1]), c2, nl2), x0, x1);
          float p0 = ex2(x0), p1 = ex2(x1);
          if (diag) {  // key j*128 + k is visible to query row r only if k <= r
            const int kk = CW * g + e;
            if (kk > r) p0 = 0.f;
            if (kk + 1 > r) p1 = 0.f;
          }
          pk[e / 2] = pack_bf16(p0, p1);
        }
      }
      ok = mbar_wait(bar_dp_full, j & 1, abort_flag, 0x1602);
      if (!ok) break;
      tc_fence_after();
      uint32_t dk[CW / 2];
      {
        float dp[CW];
        tmem_ld32(lane_base + C::COL_DP + CW * g, dp);
#pragma unroll
        for (int e = 0; e < CW; e += 2) {
          const unsigned long long pp = f2(__uint_as_float(pk[e / 2] << 16), __uint_as_float(pk[e / 2] & 0xFFFF0000u));
          float s0, s1;
          f2_split(f2_mul(pp, f2_add(f2(dp[e], dp[e + 1]), nd2)), s0, s1);
          dk[e / 2] = pack_bf16(s0, s1);
        }
      }
      if (j > 0) {  // dQ += dS_{j-1} K_{j-1} has finished reading the dS tile
        ok = mbar_wait(bar_dsm_free, (j - 1) & 1, abort_flag, 0x1603);
        if (!ok) break;
      }
#pragma unroll
      for (int u = 0; u < CW / 8; ++u) {
        const uint32_t off = sw128_offset(r, (CW / 8) * g + u);
        *reinterpret_cast<uint4*>(ds_base + off) = make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar_ds_ready);
    }
    if (ok) ok = mbar_wait(bar_dq_done, 0, abort_flag, 0x1604);
    if (ok) {
      // group g stores d columns [g D/4, (g+1) D/4) of scale * dQ (the TMEM load
      // is warp-collective, so padding rows load too and only skip the store)
      constexpr int DW = D / C::NWG;
      tc_fence_after();
      float v[DW];
      if constexpr (DW == 32)
        tmem_ld32(lane_base + C::COL_DQ + DW * g, v);
      else
        tmem_ld16(lane_base + C::COL_DQ + DW * g, v);
      if (qrow < p.N) {
        uint4 o[DW / 8];
        uint32_t* ou = reinterpret_cast<uint32_t*>(o);
#pragma unroll
        for (int e = 0; e < DW / 2; ++e) ou[e] = pack_bf16(v[2 * e] * p.scale, v[2 * e + 1] * p.scale);
        uint4* dst = reinterpret_cast<uint4*>(p.dq + (static_cast<size_t>(bh) * p.N + qrow) * D + DW * g);
#pragma unroll
        for (int e = 0; e < DW / 8; ++e) dst[e] = o[e];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::WARP_MMA) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace fa2
