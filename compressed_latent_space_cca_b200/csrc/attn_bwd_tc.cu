// Causal attention backward on tcgen05 / TMEM / TMA for sm_100a: head_dim 128, fp16 q, k, v and
// dO, fp32 softmax statistics and accumulation.
//
// "Compressed Convolutional Attention" (gist.science/es/paper/2510.04476, section 4 times the
// backward of CCGQA; section 2.C: one K/V head per group of G query heads). With
// P = softmax(scale q k^T) over the keys at or before each query and dO = dL/dO:
//   dV = P^T dO,  dP = dO V^T,  dS = P o (dP - delta),  delta_t = sum_i dO[t,i] O[t,i],
//   dQ = scale dS K,  dK = scale dS^T Q,
// with dK and dV summed over the query heads of a group. P is recomputed from q, k and the
// base-2 log-sum-exp of each row that the forward attention kernel leaves: P = 2^(c q.k - lse2),
// c = scale log2(e).
//
// Two kernels, so that no dQ sums cross CTAs:
//  dq kernel (query-stationary): a CTA per (sequence, query head, 128-query tile) walks the 128-key
//   blocks at or before the diagonal. S = Q K_j^T (two TMEM slots) and dP = dO V_j^T (one slot, freed
//   as soon as the softmax warps have read it) go to TMEM; the softmax warps turn each pair into dS
//   (fp16), written over S; dQ += dS K_j (A from TMEM, K_j read MN-major) accumulates in TMEM; the
//   epilogue scales and stores dQ. 128-key blocks keep every MMA at N = 128 or K = 128: the MMAs
//   are issued by one lane at a rate that N = 64 products would not keep up with.
//  dkv kernel (key-stationary): a CTA per (sequence, KV group, 128-key tile, chunk of up to
//   kUnitsPerChunk (64-query block, head) units) holds K and V and walks its units. S^T = K Q_i^T
//   and dP^T = V dO_i^T go to TMEM; the softmax warps write P^T and dS^T (fp16) over them in TMEM,
//   where they are the A operands of dV += P^T dO_i and dK += dS^T Q_i (Q_i and dO_i read
//   MN-major); the epilogue adds the chunk's dK (scaled) and dV to fp32 sums with vector atomics,
//   so that the long key tiles near the start of a sequence can be split over several CTAs.
// Both: warp 0 issues the TMA loads, warp 1 the MMAs (an elected lane each); the other warps do the
// softmax and the epilogue, two (dq) or four (dkv) per TMEM lane quadrant (warp w reads lanes
// 32 (w % 4) ..), one row per thread, each taking its share of the row's columns. Two TMEM slots let
// the softmax of one unit overlap the MMAs of its neighbours, and the load rings (three K/V stages,
// four Q/dO slots) keep the next units' operands in flight. Every mbarrier wait is bounded.
#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

constexpr int D = 128;
// softmax / epilogue warps of each kernel and the columns of a 64-column block each one takes
// (the dq kernel's 128-key blocks, the dkv kernel's 64-query units)
constexpr int DQ_SM_WARPS = 16, KV_SM_WARPS = 16;
constexpr int DQ_THREADS = 64 + 32 * DQ_SM_WARPS, KV_THREADS = 64 + 32 * KV_SM_WARPS;
constexpr int DQ_COLS = 128 / (DQ_SM_WARPS / 4), KV_COLS = 64 / (KV_SM_WARPS / 4);
constexpr int TMEM_COLS = 512;
constexpr int SW = 128;  // bytes of one swizzled row (64 fp16)

// ---- dq kernel geometry ----
constexpr int DQ_QT = 128;                        // queries per tile
constexpr int DQ_KB = 128;                        // keys per block
constexpr int DQ_K_STAGES = 3, DQ_V_STAGES = 2;  // V is released when dP has read it, K after dQ
constexpr int DQ_TILE_HALF = DQ_QT * SW;          // 16 KB: 128 rows x 64 columns
constexpr int DQ_KV_HALF = DQ_KB * SW;            // 16 KB: 128 rows x 64 columns
constexpr int DQ_OFF_Q = 0;
constexpr int DQ_OFF_DO = DQ_OFF_Q + 2 * DQ_TILE_HALF;
constexpr int DQ_OFF_K = DQ_OFF_DO + 2 * DQ_TILE_HALF;
constexpr int DQ_OFF_V = DQ_OFF_K + DQ_K_STAGES * 2 * DQ_KV_HALF;
constexpr int DQ_OFF_BAR = DQ_OFF_V + DQ_V_STAGES * 2 * DQ_KV_HALF;
constexpr size_t DQ_SMEM = DQ_OFF_BAR + 256 + 1024;
constexpr uint32_t DQ_COL_S = 0, DQ_COL_DP = 256, DQ_COL_DQ = 384;  // S[s] at +128 s, one dP

// ---- dkv kernel geometry ----
constexpr int KV_KT = 128;                        // keys per tile
constexpr int KV_QB = 64;                         // queries per unit
constexpr int KV_TILE_HALF = KV_KT * SW;          // 16 KB
constexpr int KV_Q_HALF = KV_QB * SW;             // 8 KB
constexpr int KV_OFF_K = 0;
constexpr int KV_OFF_V = KV_OFF_K + 2 * KV_TILE_HALF;
constexpr int KV_QSLOTS = 4;                               // load ring depth
constexpr int KV_OFF_Q = KV_OFF_V + 2 * KV_TILE_HALF;      // [slots][2 halves]
constexpr int KV_OFF_DO = KV_OFF_Q + KV_QSLOTS * 2 * KV_Q_HALF;
constexpr int KV_OFF_LSE = KV_OFF_DO + KV_QSLOTS * 2 * KV_Q_HALF;  // [slots][64] fp32
constexpr int KV_OFF_DELTA = KV_OFF_LSE + KV_QSLOTS * KV_QB * 4;   // [slots][64] fp32
constexpr int KV_OFF_BAR = KV_OFF_DELTA + KV_QSLOTS * KV_QB * 4;
constexpr size_t KV_SMEM = KV_OFF_BAR + 256 + 1024;
// St[s], dPt[s] at +64 s; P^T and dS^T (fp16 pairs) overlay them, each softmax warp's 16 queries in
// the first 8 of its own 16 columns
constexpr uint32_t KV_COL_ST = 0, KV_COL_DPT = 128, KV_COL_DV = 256, KV_COL_DK = 384;
// units per CTA: fewer CTAs pay fewer K/V loads and dK/dV reductions; measured at S = 16384 (backward
// ms): 24 -> 2.21, 32 -> 2.17, 48 -> 2.06, 96 -> 2.02, 128 -> 2.04, 192 -> 2.02, 256 -> 2.01
constexpr int kUnitsPerChunk = 96;
static_assert(DQ_SMEM <= 232448 && KV_SMEM <= 232448, "shared memory of one CTA");

struct BwdMaps {
  CUtensorMap q, dO, k, v;  // dq kernel: q, dO boxes 64 x 128 rows, k, v 64 x 64; dkv kernel: the reverse
};

struct BwdParams {
  int B, S, nq, nkv, G;
  int Lq, Lkv;
  int Sp;            // row stride of lse2 / delta per (sequence, head)
  float scale, c2;   // softmax scale and scale * log2(e)
  const float* lse2;   // [B][nq][Sp]
  const float* delta;  // [B][nq][Sp]
  float* dq;           // [B, S, Lq]  dq kernel: written
  float* dk;           // [B, S, Lkv] dkv kernel: added to
  float* dv;           // [B, S, Lkv] dkv kernel: added to
  unsigned* err;
  // dkv kernel: chunks per (sequence, group) and key tiles per sequence
  int nkt, chunks;
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 32 lanes x 16 columns of 32-bit: thread i stores r[0..15] to lane (base + i), columns [col, col + 16)
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32"
      " [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// 16-byte units of the K-step offset kk (16 elements) inside a K-major swizzled tile whose two
// 64-column halves lie `half` bytes apart
__device__ __forceinline__ uint32_t kmaj_step(int kk, int half) {
  return (uint32_t)(((kk >> 2) * half + (kk & 3) * 32) >> 4);
}

// ============================================================ dq kernel ==
__global__ void __launch_bounds__(DQ_THREADS, 1) attn_bwd_dq_kernel(const __grid_constant__ BwdMaps maps,
                                                                     const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DQ_OFF_BAR);
  uint64_t* q_full = bars;                        // Q and dO of the tile
  uint64_t* k_full = bars + 1;                    // [DQ_K_STAGES]
  uint64_t* k_empty = k_full + DQ_K_STAGES;       // [DQ_K_STAGES]
  uint64_t* v_full = k_empty + DQ_K_STAGES;       // [DQ_V_STAGES]
  uint64_t* v_empty = v_full + DQ_V_STAGES;       // [DQ_V_STAGES]
  uint64_t* st_full = v_empty + DQ_V_STAGES;      // [2] S and dP of a block in TMEM
  uint64_t* ds_full = st_full + 2;                // [2] dS written over S (every softmax warp)
  uint64_t* dp_free = ds_full + 2;                // dP read by every softmax warp
  uint64_t* dq_full = dp_free + 1;                // dQ complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dq_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // tile: longest (last query tiles) first
  const int nqt = (p.S + DQ_QT - 1) / DQ_QT;
  const int bh = blockIdx.x % (p.B * p.nq);
  const int qt = nqt - 1 - blockIdx.x / (p.B * p.nq);
  const int b = bh / p.nq, h = bh % p.nq, g = h / p.G;
  const int q_last = min(qt * DQ_QT + DQ_QT - 1, p.S - 1);
  const int nkb = q_last / DQ_KB + 1;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < DQ_K_STAGES; ++s) {
      mbar_init(smem_u32(&k_full[s]), 1);
      mbar_init(smem_u32(&k_empty[s]), 1);
    }
    for (int s = 0; s < DQ_V_STAGES; ++s) {
      mbar_init(smem_u32(&v_full[s]), 1);
      mbar_init(smem_u32(&v_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&st_full[s]), 1);
      mbar_init(smem_u32(&ds_full[s]), DQ_SM_WARPS);
    }
    mbar_init(smem_u32(dp_free), DQ_SM_WARPS);
    mbar_init(smem_u32(dq_full), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.dO);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA --
    if (elect_one_sync()) mbar_arrive_expect_tx(smem_u32(q_full), 4 * DQ_TILE_HALF);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      if (elect_one_sync())
        tma_load_3d(smem_u32(smem + DQ_OFF_Q + hf * DQ_TILE_HALF), &maps.q, smem_u32(q_full), h * D + hf * 64,
                    qt * DQ_QT, b);
      if (elect_one_sync())
        tma_load_3d(smem_u32(smem + DQ_OFF_DO + hf * DQ_TILE_HALF), &maps.dO, smem_u32(q_full), h * D + hf * 64,
                    qt * DQ_QT, b);
    }
    for (int j = 0; j < nkb; ++j) {
      const int sk = j % DQ_K_STAGES, sv = j % DQ_V_STAGES;
      if (!mbar_wait_bounded(smem_u32(&k_empty[sk]), ((j / DQ_K_STAGES) & 1) ^ 1, p.err, abort_flag,
                             wait_site(kSiteAttnBwd, 1, 1)))
        break;
      if (elect_one_sync()) mbar_arrive_expect_tx(smem_u32(&k_full[sk]), 2 * DQ_KV_HALF);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
        if (elect_one_sync())
          tma_load_3d(smem_u32(smem + DQ_OFF_K + (sk * 2 + hf) * DQ_KV_HALF), &maps.k, smem_u32(&k_full[sk]),
                      g * D + hf * 64, j * DQ_KB, b);
      if (!mbar_wait_bounded(smem_u32(&v_empty[sv]), ((j / DQ_V_STAGES) & 1) ^ 1, p.err, abort_flag,
                             wait_site(kSiteAttnBwd, 1, 7)))
        break;
      if (elect_one_sync()) mbar_arrive_expect_tx(smem_u32(&v_full[sv]), 2 * DQ_KV_HALF);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
        if (elect_one_sync())
          tma_load_3d(smem_u32(smem + DQ_OFF_V + (sv * 2 + hf) * DQ_KV_HALF), &maps.v, smem_u32(&v_full[sv]),
                      g * D + hf * 64, j * DQ_KB, b);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA --
    const uint32_t idesc_s = idesc_f32acc(DQ_QT, DQ_KB, 0, 0, kFmtF16);  // Q, K (dO, V) K-major
    const uint32_t idesc_dq = idesc_f32acc(DQ_QT, D, 0, 1, kFmtF16);     // dS from TMEM, K MN-major
    const uint32_t sw_hi = desc_hi(smem_desc_sw128(smem_u32(smem), 16, 1024));
    const uint32_t mn_hi = desc_hi(smem_desc_sw128(smem_u32(smem), DQ_KV_HALF, 1024));
    const uint32_t q_lo = desc_lo(smem_desc_sw128(smem_u32(smem + DQ_OFF_Q), 16, 1024));
    const uint32_t do_lo = desc_lo(smem_desc_sw128(smem_u32(smem + DQ_OFF_DO), 16, 1024));
    const uint32_t k_lo = desc_lo(smem_desc_sw128(smem_u32(smem + DQ_OFF_K), 16, 1024));
    const uint32_t v_lo = desc_lo(smem_desc_sw128(smem_u32(smem + DQ_OFF_V), 16, 1024));
    const uint32_t kmn_lo = desc_lo(smem_desc_sw128(smem_u32(smem + DQ_OFF_K), DQ_KV_HALF, 1024));
    constexpr uint32_t kStageStep = (2 * DQ_KV_HALF) >> 4;
    if (!mbar_wait_bounded(smem_u32(q_full), 0, p.err, abort_flag, wait_site(kSiteAttnBwd, 2, 2))) goto done;
    tc_fence_after();
    for (int j = 0; j <= nkb; ++j) {
      if (j < nkb) {
        const int sk = j % DQ_K_STAGES, sv = j % DQ_V_STAGES, s = j & 1;
        if (!mbar_wait_bounded(smem_u32(&k_full[sk]), (j / DQ_K_STAGES) & 1, p.err, abort_flag,
                               wait_site(kSiteAttnBwd, 2, 3)))
          goto done;
        tc_fence_after();
        // S[s] = Q K_j^T: slot s was last read by the softmax of block j - 2, whose ds_full this loop
        // waited for at j - 1, and by the dQ MMA of block j - 2 issued before
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          if (elect_one_sync())
            umma_ss_lohi(tmem + DQ_COL_S + 128 * s, q_lo + kmaj_step(kk, DQ_TILE_HALF), sw_hi,
                         k_lo + sk * kStageStep + kmaj_step(kk, DQ_KV_HALF), sw_hi, idesc_s, kk > 0);
        // dP = dO V_j^T into the one dP slot, once the softmax warps have read block j - 1's
        if (j >= 1 && !mbar_wait_bounded(smem_u32(dp_free), (j - 1) & 1, p.err, abort_flag,
                                         wait_site(kSiteAttnBwd, 2, 5)))
          goto done;
        if (!mbar_wait_bounded(smem_u32(&v_full[sv]), (j / DQ_V_STAGES) & 1, p.err, abort_flag,
                               wait_site(kSiteAttnBwd, 2, 6)))
          goto done;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          if (elect_one_sync())
            umma_ss_lohi(tmem + DQ_COL_DP, do_lo + kmaj_step(kk, DQ_TILE_HALF), sw_hi,
                         v_lo + sv * kStageStep + kmaj_step(kk, DQ_KV_HALF), sw_hi, idesc_s, kk > 0);
        if (elect_one_sync()) umma_commit(smem_u32(&st_full[s]));
        if (elect_one_sync()) umma_commit(smem_u32(&v_empty[sv]));  // V_j is read by dP alone
      }
      if (j >= 1) {
        const int jp = j - 1, sp = jp & 1, skp = jp % DQ_K_STAGES;
        if (!mbar_wait_bounded(smem_u32(&ds_full[sp]), (jp >> 1) & 1, p.err, abort_flag,
                               wait_site(kSiteAttnBwd, 2, 4)))
          goto done;
        tc_fence_after();
        // dQ += dS K_jp: A = dS (fp16 pairs: keys 16 kk .. 16 kk + 15 in the 8 columns from
        // DQ_COLS (kk / 2) + 8 (kk % 2) of S[sp], each softmax warp's packed share at the start of its
        // own columns), B = K_jp read as [d x keys] MN-major (LBO = the 64-column half, SBO = 8 keys)
        static_assert(DQ_COLS == 32, "two 16-key MMA steps per softmax warp's share");
#pragma unroll
        for (int kk = 0; kk < DQ_KB / 16; ++kk)
          if (elect_one_sync())
            umma_ts_lohi(tmem + DQ_COL_DQ, tmem + DQ_COL_S + 128 * sp + DQ_COLS * (kk >> 1) + 8 * (kk & 1),
                         kmn_lo + skp * kStageStep + ((kk * 16 * SW) >> 4), mn_hi, idesc_dq, jp > 0 || kk > 0);
        if (elect_one_sync()) umma_commit(smem_u32(&k_empty[skp]));
      }
    }
    if (elect_one_sync()) umma_commit(smem_u32(dq_full));
  } else {
    // ------------------------------------------------------------ softmax --
    const int quad = warp & 3;
    const int part = (warp - 2) >> 2;  // this warp's DQ_COLS of the block's 128 keys
    const int r = quad * 32 + lane;
    const int t = qt * DQ_QT + r;
    const bool row_ok = t < p.S;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const size_t srow = ((size_t)b * p.nq + h) * p.Sp;
    const float lse2 = row_ok ? p.lse2[srow + t] : 0.f;
    const float dl = row_ok ? p.delta[srow + t] : 0.f;
    const float c2 = p.c2;
    bool bad = false;
    for (int j = 0; j < nkb; ++j) {
      const int s = j & 1;
      if (!mbar_wait_bounded(smem_u32(&st_full[s]), (j >> 1) & 1, p.err, abort_flag, wait_site(kSiteAttnBwd, 3, 5)))
        goto done;
      tc_fence_after();
      static_assert(DQ_COLS == 32, "the dq softmax reads 32 columns a warp");
      uint32_t sv[DQ_COLS], dp[DQ_COLS];
      tmem_ld_32x32b_x32(tmem + lane_off + DQ_COL_S + 128 * s + DQ_COLS * part, sv);
      tmem_ld_32x32b_x32(tmem + lane_off + DQ_COL_DP + DQ_COLS * part, dp);
      tmem_ld_wait();
      tc_fence_before();  // dP may take the next block's product
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(dp_free));
      const int key0 = j * DQ_KB + DQ_COLS * part;
      uint32_t pk[DQ_COLS / 2];
      float dmax = 0.f;  // largest |dS| of the block, checked against the fp16 range once
      // every key of the warp's share visible to every row of the warp: the choice is warp-uniform, so
      // the warp stays converged for the tcgen05.st that follows
      if (__all_sync(0xffffffffu, row_ok && key0 + DQ_COLS - 1 <= t)) {
#pragma unroll
        for (int c = 0; c < DQ_COLS; c += 2) {
          const float d0 = fast_exp2(fmaf(u2f(sv[c]), c2, -lse2)) * (u2f(dp[c]) - dl);
          const float d1 = fast_exp2(fmaf(u2f(sv[c + 1]), c2, -lse2)) * (u2f(dp[c + 1]) - dl);
          dmax = fmaxf(dmax, fmaxf(fabsf(d0), fabsf(d1)));
          pk[c >> 1] = pack_f16x2(d0, d1);
        }
      } else {
#pragma unroll
        for (int c = 0; c < DQ_COLS; c += 2) {
          float ds[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool vis = row_ok && key0 + c + e <= t;
            const float pr = vis ? fast_exp2(fmaf(u2f(sv[c + e]), c2, -lse2)) : 0.f;
            ds[e] = vis ? pr * (u2f(dp[c + e]) - dl) : 0.f;
            dmax = fmaxf(dmax, fabsf(ds[e]));
          }
          pk[c >> 1] = pack_f16x2(ds[0], ds[1]);
        }
      }
      bad |= f16_overflow(dmax);
      // the warp's keys 2c, 2c + 1 go to packed column c of its own share of S[s] (the first half of
      // the columns this warp has just read): another warp's unread scores are never overwritten
      tmem_st_32x32b_x16(tmem + lane_off + DQ_COL_S + 128 * s + DQ_COLS * part, pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ds_full[s]));
    }
    report_range(bad, p.err);
    if (!mbar_wait_bounded(smem_u32(dq_full), 0, p.err, abort_flag, wait_site(kSiteAttnBwd, 3, 6))) goto done;
    tc_fence_after();
    float* out = p.dq + ((size_t)b * p.S + t) * p.Lq + h * D;
#pragma unroll 1
    for (int c4 = part; c4 < part + 1; ++c4) {  // 32 of the 128 columns per warp
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + lane_off + DQ_COL_DQ + 32 * c4, v);
      tmem_ld_wait();
      if (row_ok) {
#pragma unroll
        for (int m = 0; m < 8; ++m)
          *reinterpret_cast<float4*>(out + 32 * c4 + 4 * m) =
              make_float4(u2f(v[4 * m]) * p.scale, u2f(v[4 * m + 1]) * p.scale, u2f(v[4 * m + 2]) * p.scale,
                          u2f(v[4 * m + 3]) * p.scale);
      }
    }
    tc_fence_before();
  }
done:
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// =========================================================== dkv kernel ==
struct KvItem {
  int b, g, kt, u0, u1, nqb0;  // units [u0, u1) of key tile kt; unit u: query block nqb0 + u / G, head u % G
};

__device__ __forceinline__ KvItem kv_item(const BwdParams& p, int w) {
  KvItem it;
  const int bg = w % (p.B * p.nkv);
  int c = w / (p.B * p.nkv);
  it.b = bg / p.nkv;
  it.g = bg % p.nkv;
  const int nqb = (p.S + KV_QB - 1) / KV_QB;
  int kt = 0;
  for (; kt < p.nkt; ++kt) {  // chunks of the longest key tiles first
    const int U = p.G * (nqb - 2 * kt);
    const int ch = (U + kUnitsPerChunk - 1) / kUnitsPerChunk;
    if (c < ch) {
      it.u0 = c * kUnitsPerChunk;
      it.u1 = min(U, it.u0 + kUnitsPerChunk);
      break;
    }
    c -= ch;
  }
  it.kt = kt;
  it.nqb0 = 2 * kt;
  return it;
}

__global__ void __launch_bounds__(KV_THREADS, 1) attn_bwd_dkv_kernel(const __grid_constant__ BwdMaps maps,
                                                                      const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + KV_OFF_BAR);
  uint64_t* kv_full = bars;            // K and V of the tile
  uint64_t* qd_full = bars + 1;                // [KV_QSLOTS] Q_i, dO_i, lse2, delta of a unit
  uint64_t* qd_empty = qd_full + KV_QSLOTS;    // [KV_QSLOTS]
  uint64_t* st_full = qd_empty + KV_QSLOTS;    // [2] S^T, dP^T in TMEM
  uint64_t* p_full = st_full + 2;      // [2] P^T, dS^T written over them (every softmax warp)
  uint64_t* acc_full = p_full + 2;     // dK, dV complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const KvItem it = kv_item(p, blockIdx.x);
  const int n_units = it.u1 - it.u0;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(kv_full), 1);
    for (int s = 0; s < KV_QSLOTS; ++s) {
      mbar_init(smem_u32(&qd_full[s]), 1);
      mbar_init(smem_u32(&qd_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&st_full[s]), 1);
      mbar_init(smem_u32(&p_full[s]), KV_SM_WARPS);
    }
    mbar_init(smem_u32(acc_full), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.dO);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA --
    if (elect_one_sync()) mbar_arrive_expect_tx(smem_u32(kv_full), 4 * KV_TILE_HALF);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      if (elect_one_sync())
        tma_load_3d(smem_u32(smem + KV_OFF_K + hf * KV_TILE_HALF), &maps.k, smem_u32(kv_full), it.g * D + hf * 64,
                    it.kt * KV_KT, it.b);
      if (elect_one_sync())
        tma_load_3d(smem_u32(smem + KV_OFF_V + hf * KV_TILE_HALF), &maps.v, smem_u32(kv_full), it.g * D + hf * 64,
                    it.kt * KV_KT, it.b);
    }
    for (int n = 0; n < n_units; ++n) {
      const int u = it.u0 + n, s = n % KV_QSLOTS;
      const int qb = it.nqb0 + u / p.G, h = it.g * p.G + u % p.G;
      if (!mbar_wait_bounded(smem_u32(&qd_empty[s]), ((n / KV_QSLOTS) & 1) ^ 1, p.err, abort_flag,
                             wait_site(kSiteAttnBwd, 4, 1)))
        break;
      if (elect_one_sync()) mbar_arrive_expect_tx(smem_u32(&qd_full[s]), 4 * KV_Q_HALF + 2 * KV_QB * 4);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        if (elect_one_sync())
          tma_load_3d(smem_u32(smem + KV_OFF_Q + (s * 2 + hf) * KV_Q_HALF), &maps.q, smem_u32(&qd_full[s]),
                      h * D + hf * 64, qb * KV_QB, it.b);
        if (elect_one_sync())
          tma_load_3d(smem_u32(smem + KV_OFF_DO + (s * 2 + hf) * KV_Q_HALF), &maps.dO, smem_u32(&qd_full[s]),
                      h * D + hf * 64, qb * KV_QB, it.b);
      }
      const size_t srow = ((size_t)it.b * p.nq + h) * p.Sp + (size_t)qb * KV_QB;
      if (elect_one_sync()) {
        bulk_load(smem_u32(smem + KV_OFF_LSE + s * KV_QB * 4), p.lse2 + srow, KV_QB * 4, smem_u32(&qd_full[s]));
        bulk_load(smem_u32(smem + KV_OFF_DELTA + s * KV_QB * 4), p.delta + srow, KV_QB * 4, smem_u32(&qd_full[s]));
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA --
    const uint32_t idesc_st = idesc_f32acc(KV_KT, KV_QB, 0, 0, kFmtF16);  // K (V) and Q (dO) K-major
    const uint32_t idesc_acc = idesc_f32acc(KV_KT, D, 0, 1, kFmtF16);     // P^T (dS^T) from TMEM, dO (Q) MN-major
    const uint32_t sw_hi = desc_hi(smem_desc_sw128(smem_u32(smem), 16, 1024));
    const uint32_t mn_hi = desc_hi(smem_desc_sw128(smem_u32(smem), KV_Q_HALF, 1024));
    const uint32_t k_lo = desc_lo(smem_desc_sw128(smem_u32(smem + KV_OFF_K), 16, 1024));
    const uint32_t v_lo = desc_lo(smem_desc_sw128(smem_u32(smem + KV_OFF_V), 16, 1024));
    const uint32_t q_lo = desc_lo(smem_desc_sw128(smem_u32(smem + KV_OFF_Q), 16, 1024));
    const uint32_t do_lo = desc_lo(smem_desc_sw128(smem_u32(smem + KV_OFF_DO), 16, 1024));
    const uint32_t qmn_lo = desc_lo(smem_desc_sw128(smem_u32(smem + KV_OFF_Q), KV_Q_HALF, 1024));
    const uint32_t domn_lo = desc_lo(smem_desc_sw128(smem_u32(smem + KV_OFF_DO), KV_Q_HALF, 1024));
    constexpr uint32_t kQSlot = (2 * KV_Q_HALF) >> 4;
    if (!mbar_wait_bounded(smem_u32(kv_full), 0, p.err, abort_flag, wait_site(kSiteAttnBwd, 5, 2))) goto done;
    tc_fence_after();
    for (int n = 0; n <= n_units; ++n) {
      if (n < n_units) {
        const int s = n & 1, q = n % KV_QSLOTS;  // TMEM slot, load slot
        if (!mbar_wait_bounded(smem_u32(&qd_full[q]), (n / KV_QSLOTS) & 1, p.err, abort_flag,
                               wait_site(kSiteAttnBwd, 5, 3)))
          goto done;
        tc_fence_after();
        // S^T[s] = K Q_i^T, dP^T[s] = V dO_i^T; slot s was last read by the softmax of unit n - 2,
        // whose p_full this loop waited for at n - 1, and by the dV / dK MMAs of unit n - 2 issued
        // before (tcgen05 MMAs of one thread run in order)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          if (elect_one_sync())
            umma_ss_lohi(tmem + KV_COL_ST + 64 * s, k_lo + kmaj_step(kk, KV_TILE_HALF), sw_hi,
                         q_lo + q * kQSlot + kmaj_step(kk, KV_Q_HALF), sw_hi, idesc_st, kk > 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          if (elect_one_sync())
            umma_ss_lohi(tmem + KV_COL_DPT + 64 * s, v_lo + kmaj_step(kk, KV_TILE_HALF), sw_hi,
                         do_lo + q * kQSlot + kmaj_step(kk, KV_Q_HALF), sw_hi, idesc_st, kk > 0);
        if (elect_one_sync()) umma_commit(smem_u32(&st_full[s]));
      }
      if (n >= 1) {
        const int np = n - 1, sp = np & 1, qp = np % KV_QSLOTS;
        if (!mbar_wait_bounded(smem_u32(&p_full[sp]), (np >> 1) & 1, p.err, abort_flag, wait_site(kSiteAttnBwd, 5, 4)))
          goto done;
        tc_fence_after();
        // dV += P^T dO_i and dK += dS^T Q_i: A = [128 keys x 64 queries] from TMEM (fp16 pairs:
        // queries 16 kk .. 16 kk + 15 in the 8 columns from 16 kk, softmax warp kk's packed share), B =
        // dO_i / Q_i read as [d x queries] MN-major; 16 queries per MMA
        static_assert(KV_COLS == 16, "one 16-query MMA step per softmax warp's share");
#pragma unroll
        for (int kk = 0; kk < KV_QB / 16; ++kk) {
          const uint32_t bstep = (uint32_t)((kk * 16 * SW) >> 4);
          if (elect_one_sync())
            umma_ts_lohi(tmem + KV_COL_DV, tmem + KV_COL_ST + 64 * sp + KV_COLS * kk, domn_lo + qp * kQSlot + bstep,
                         mn_hi, idesc_acc, np > 0 || kk > 0);
          if (elect_one_sync())
            umma_ts_lohi(tmem + KV_COL_DK, tmem + KV_COL_DPT + 64 * sp + KV_COLS * kk, qmn_lo + qp * kQSlot + bstep,
                         mn_hi, idesc_acc, np > 0 || kk > 0);
        }
        if (elect_one_sync()) umma_commit(smem_u32(&qd_empty[qp]));
      }
    }
    if (elect_one_sync()) umma_commit(smem_u32(acc_full));
  } else {
    // ------------------------------------------------------------ softmax --
    const int quad = warp & 3;
    const int part = (warp - 2) >> 2;  // this warp's KV_COLS of a unit's 64 queries
    const int r = quad * 32 + lane;
    const int key = it.kt * KV_KT + r;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float c2 = p.c2;
    bool bad = false;
    for (int n = 0; n < n_units; ++n) {
      const int u = it.u0 + n, s = n & 1, q = n % KV_QSLOTS;
      const int q0 = (it.nqb0 + u / p.G) * KV_QB;
      if (!mbar_wait_bounded(smem_u32(&st_full[s]), (n >> 1) & 1, p.err, abort_flag, wait_site(kSiteAttnBwd, 6, 5)))
        goto done;
      tc_fence_after();
      static_assert(KV_COLS == 16, "the dkv softmax reads 16 columns a warp");
      uint32_t sv[KV_COLS], dp[KV_COLS];
      tmem_ld_32x32b_x16(tmem + lane_off + KV_COL_ST + 64 * s + KV_COLS * part, sv);
      tmem_ld_32x32b_x16(tmem + lane_off + KV_COL_DPT + 64 * s + KV_COLS * part, dp);
      tmem_ld_wait();
      // lse2 and delta of this unit came by bulk copy: observe its completion here too (the slot
      // cannot be refilled before this warp's p_full, so this is the unit's own phase)
      if (!mbar_wait_bounded(smem_u32(&qd_full[q]), (n / KV_QSLOTS) & 1, p.err, abort_flag,
                             wait_site(kSiteAttnBwd, 6, 8)))
        goto done;
      const float* lse_s = reinterpret_cast<const float*>(smem + KV_OFF_LSE + q * KV_QB * 4);
      const float* del_s = reinterpret_cast<const float*>(smem + KV_OFF_DELTA + q * KV_QB * 4);
      uint32_t pp[KV_COLS / 2], dd[KV_COLS / 2];  // this warp's queries 2c, 2c + 1 -> packed column c
      // this warp's statistics, four at a time (every lane reads the same addresses)
      float ls[KV_COLS], de[KV_COLS];
#pragma unroll
      for (int v4 = 0; v4 < KV_COLS / 4; ++v4) {
        const float4 a = *reinterpret_cast<const float4*>(lse_s + KV_COLS * part + 4 * v4);
        const float4 b = *reinterpret_cast<const float4*>(del_s + KV_COLS * part + 4 * v4);
        ls[4 * v4] = a.x, ls[4 * v4 + 1] = a.y, ls[4 * v4 + 2] = a.z, ls[4 * v4 + 3] = a.w;
        de[4 * v4] = b.x, de[4 * v4 + 1] = b.y, de[4 * v4 + 2] = b.z, de[4 * v4 + 3] = b.w;
      }
      const int qa = q0 + KV_COLS * part;  // this warp's first query
      float dmax = 0.f;  // largest |dS|, checked against the fp16 range once
      // every query of the share sees every key row of the warp: the choice is warp-uniform, so the warp
      // stays converged for the tcgen05.st that follows
      if (__all_sync(0xffffffffu, key <= qa && qa + KV_COLS - 1 < p.S)) {
#pragma unroll
        for (int c2i = 0; c2i < KV_COLS / 2; ++c2i) {
          const int c = 2 * c2i;
          const float p0 = fast_exp2(fmaf(u2f(sv[c]), c2, -ls[c]));
          const float p1 = fast_exp2(fmaf(u2f(sv[c + 1]), c2, -ls[c + 1]));
          const float d0 = p0 * (u2f(dp[c]) - de[c]), d1 = p1 * (u2f(dp[c + 1]) - de[c + 1]);
          dmax = fmaxf(dmax, fmaxf(fabsf(d0), fabsf(d1)));
          pp[c2i] = pack_f16x2(p0, p1);
          dd[c2i] = pack_f16x2(d0, d1);
        }
      } else {
#pragma unroll
        for (int c2i = 0; c2i < KV_COLS / 2; ++c2i) {
          float pv[2], dv[2];
#pragma unroll
          for (int f = 0; f < 2; ++f) {
            const int cl = 2 * c2i + f;  // column within this warp's share
            const int t = qa + cl;
            const bool vis = key <= t && t < p.S;
            const float pr = vis ? fast_exp2(fmaf(u2f(sv[cl]), c2, -ls[cl])) : 0.f;
            pv[f] = pr;
            dv[f] = vis ? pr * (u2f(dp[cl]) - de[cl]) : 0.f;
            dmax = fmaxf(dmax, fabsf(dv[f]));
          }
          pp[c2i] = pack_f16x2(pv[0], pv[1]);
          dd[c2i] = pack_f16x2(dv[0], dv[1]);
        }
      }
      bad |= f16_overflow(dmax);
      // P^T over S^T[s] and dS^T over dP^T[s], each at the start of this warp's own share of the
      // columns (read above): another warp's unread values are never overwritten
      tmem_st_32x32b_x8(tmem + lane_off + KV_COL_ST + 64 * s + KV_COLS * part, pp);
      tmem_st_32x32b_x8(tmem + lane_off + KV_COL_DPT + 64 * s + KV_COLS * part, dd);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&p_full[s]));
    }
    report_range(bad, p.err);
    if (!mbar_wait_bounded(smem_u32(acc_full), 0, p.err, abort_flag, wait_site(kSiteAttnBwd, 6, 7))) goto done;
    tc_fence_after();
    const bool key_ok = key < p.S;
    const size_t orow = ((size_t)it.b * p.S + key) * p.Lkv + it.g * D;
#pragma unroll 1
    for (int c4 = part; c4 < part + 1; ++c4) {  // 32 of the 128 columns per warp
      uint32_t v[32], k[32];
      tmem_ld_32x32b_x32(tmem + lane_off + KV_COL_DV + 32 * c4, v);
      tmem_ld_32x32b_x32(tmem + lane_off + KV_COL_DK + 32 * c4, k);
      tmem_ld_wait();
      if (key_ok) {
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          red_add_v4(p.dv + orow + 32 * c4 + 4 * m, u2f(v[4 * m]), u2f(v[4 * m + 1]), u2f(v[4 * m + 2]),
                     u2f(v[4 * m + 3]));
          red_add_v4(p.dk + orow + 32 * c4 + 4 * m, u2f(k[4 * m]) * p.scale, u2f(k[4 * m + 1]) * p.scale,
                     u2f(k[4 * m + 2]) * p.scale, u2f(k[4 * m + 3]) * p.scale);
        }
      }
    }
    tc_fence_before();
  }
done:
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

bool encode(CUtensorMap* m, const void* ptr, uint64_t width, uint64_t S, uint64_t B, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {width, S, B};
  cuuint64_t strides[2] = {width * 2, width * S * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int kv_chunks(const BlockDims& dm, int* nkt_out) {
  const int nqb = (dm.S + KV_QB - 1) / KV_QB, nkt = (dm.S + KV_KT - 1) / KV_KT;
  int chunks = 0;
  for (int kt = 0; kt < nkt; ++kt) chunks += (dm.G * (nqb - 2 * kt) + kUnitsPerChunk - 1) / kUnitsPerChunk;
  *nkt_out = nkt;
  return chunks;
}

}  // namespace

bool attention_bwd_tc_supported(const BlockDims& dm) { return attention_tc_supported(dm); }

cudaError_t launch_attention_bwd_tc(const BlockDims& dm, const AttnBwdPtrs& a, unsigned* dev_err,
                                    cudaStream_t stream) {
  if (!attention_bwd_tc_supported(dm)) return cudaErrorInvalidValue;
  BwdParams p;
  p.B = dm.B;
  p.S = dm.S;
  p.nq = dm.nq;
  p.nkv = dm.nkv;
  p.G = dm.G;
  p.Lq = dm.Lq;
  p.Lkv = dm.Lkv;
  p.Sp = a.stat_stride;
  p.scale = dm.scale;
  p.c2 = dm.scale * 1.4426950408889634f;
  p.lse2 = a.lse2;
  p.delta = a.delta;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.err = dev_err;
  p.chunks = kv_chunks(dm, &p.nkt);
  cudaError_t e;
  {
    BwdMaps m;
    if (!encode(&m.q, a.q, dm.Lq, dm.S, dm.B, DQ_QT) || !encode(&m.dO, a.dO, dm.Lq, dm.S, dm.B, DQ_QT) ||
        !encode(&m.k, a.k, dm.Lkv, dm.S, dm.B, DQ_KB) || !encode(&m.v, a.v, dm.Lkv, dm.S, dm.B, DQ_KB))
      return cudaErrorInvalidValue;
    if ((e = cudaFuncSetAttribute(attn_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DQ_SMEM)) !=
        cudaSuccess)
      return e;
    const unsigned grid = (unsigned)(dm.B * dm.nq * ((dm.S + DQ_QT - 1) / DQ_QT));
    attn_bwd_dq_kernel<<<grid, DQ_THREADS, DQ_SMEM, stream>>>(m, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    BwdMaps m;
    if (!encode(&m.q, a.q, dm.Lq, dm.S, dm.B, KV_QB) || !encode(&m.dO, a.dO, dm.Lq, dm.S, dm.B, KV_QB) ||
        !encode(&m.k, a.k, dm.Lkv, dm.S, dm.B, KV_KT) || !encode(&m.v, a.v, dm.Lkv, dm.S, dm.B, KV_KT))
      return cudaErrorInvalidValue;
    if ((e = cudaFuncSetAttribute(attn_bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KV_SMEM)) !=
        cudaSuccess)
      return e;
    const unsigned grid = (unsigned)(dm.B * dm.nkv * p.chunks);
    attn_bwd_dkv_kernel<<<grid, KV_THREADS, KV_SMEM, stream>>>(m, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace cca
