// Causal flash attention on the compressed heads, tcgen05 / TMEM / TMA for
// sm_100a, head_dim 128, fp16 q / k / v / P / O, fp32 softmax and accumulation.
//
// "Compressed Convolutional Attention" (gist.science/es/paper/2510.04476):
// attention runs entirely in the compressed latent (section 2.A) and, in
// CCGQA, one K/V head serves a group of G query heads (section 2.C):
//   O[t, h] = sum_{s <= t} softmax_s(q[t,h] . k[s,g(h)] * scale) v[s,g(h)],
//   g(h) = h / G.
//
// One CTA owns a pair of 128-query tiles of one KV group (for G >= 2 two
// query heads at the same positions, for G = 1 two consecutive query tiles
// of one head), so every K/V tile it loads serves both. Roles:
//   warp 0      TMA, run by the whole warp with an elected lane issuing: Q
//               tiles once per pair, then K tiles (3-stage ring) and V tiles
//               (2-stage ring)
//   warp 1      the MMA loop, run by the whole warp so that its control flow
//               and descriptor arithmetic stay warp-uniform; an elected lane
//               issues tcgen05.mma: S_j = Q_j K^T (SS form) into TMEM, then
//               O_j += P_j V (TS form, P read from TMEM)
//   warps 2-17  softmax, eight warps per tile, two on each SMSP: each warp owns
//               16 query rows (half a TMEM lane quadrant) and reads its S rows
//               with the 16-lane TMEM shapes, so each thread holds 32 keys of two
//               rows and a quad of threads shares a row; they keep the
//               running max / sum, write P (fp16) back over S in TMEM, rescale
//               their O rows in TMEM when the max grows by more than 2^8, and
//               finally normalise O and store it.
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; P_j overlays
// the first 64 columns of S_j. The two tiles ping-pong: while one softmax
// group works, the tensor core runs the other tile's MMAs. Key tiles above
// the diagonal are never loaded (causal tile skipping); the diagonal tile is
// masked per element. Pairs are assigned to the persistent CTAs by a host-side
// longest-processing-time schedule (largest pair to the least-loaded CTA),
// passed in the kernel parameters. Every mbarrier wait is bounded.
#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

constexpr int D = 128;           // head dim
constexpr int TQ = 128;          // queries per tile
constexpr int TK = 128;          // keys per tile
constexpr int K_STAGES = 3, V_STAGES = 2;
constexpr int HALF_BYTES = 128 * 64 * 2;  // 128 rows x 64 fp16 (one 128-byte swizzle span)
constexpr int TILE_BYTES = 2 * HALF_BYTES;  // 128 x 128 fp16
constexpr int NUM_SOFTMAX_WARPS = 16;  // eight per query tile
constexpr int NUM_THREADS = 64 + 32 * NUM_SOFTMAX_WARPS;
constexpr int TMEM_COLS = 512;
constexpr uint32_t COL_S0 = 0, COL_O0 = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale O only if the max grows by > 2^8

// shared memory: Q0 | Q1 | K[3] | V[2] | barriers
constexpr int OFF_Q = 0;
constexpr int OFF_K = 2 * TILE_BYTES;
constexpr int OFF_V = OFF_K + K_STAGES * TILE_BYTES;
constexpr int OFF_BAR = OFF_V + V_STAGES * TILE_BYTES;
constexpr int MAX_CTAS = 160;
constexpr int MAX_LIST = 4096;  // entries a host schedule can hold in the kernel parameters
// A partial result of one 128-row tile: O as [16 chunks of 8 columns][128 rows][8] fp32 (a warp's
// accesses to one chunk cover 256 contiguous bytes per 8 rows), then the running max [128] and sum [128].
constexpr int PART_TILE = D * TQ + 2 * TQ;  // floats
constexpr size_t SMEM_BYTES = OFF_BAR + 256 + 1024;

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair, on the FMA and integer pipes, for x in [-inf, 126]:
// x = n + f with n = round(x) (adding 1.5 * 2^23 leaves n in the low mantissa
// bits) and |f| <= 1/2; 2^f from a cubic fitted to 2^f on [-1/2, 1/2] by
// iteratively reweighted least squares (max relative error 1.0e-4, below the
// fp16 rounding of P); 2^n is added to the exponent field. A share of the
// probabilities takes this path so that the special-function unit, which
// otherwise paces the tensor core at head_dim 128, does less of the work.
__device__ __forceinline__ void exp2_fma_x2(float x0, float x1, float& p0, float& p1) {
  constexpr float kMagic = 12582912.0f;
  x0 = fmaxf(x0, -126.0f);
  x1 = fmaxf(x1, -126.0f);
  float t0, t1, r0, r1, f0, f1, q0, q1;
  add2(t0, t1, x0, x1, kMagic, kMagic);
  add2(r0, r1, t0, t1, -kMagic, -kMagic);
  fma2(f0, f1, r0, r1, -1.0f, -1.0f, x0, x1);
  fma2(q0, q1, 0.05500893f, 0.05500893f, f0, f1, 0.24221097f, 0.24221097f);
  fma2(q0, q1, q0, q1, f0, f1, 0.69328290f, 0.69328290f);
  fma2(q0, q1, q0, q1, f0, f1, 1.0f, 1.0f);
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}
#ifndef CCA_POLY_EVERY
#define CCA_POLY_EVERY 4  // one pair in CCA_POLY_EVERY takes exp2_fma_x2 (0: none)
#endif

struct AttnMaps {
  CUtensorMap q, k, v;
  CUtensorMap o;  // attention output, boxes of 64 columns x 16 rows (one softmax warp's rows)
};

struct AttnParams {
  int B, S, nq, nkv, G;
  int num_qt;  // query tiles per sequence
  int pairs;   // tile pairs per (sequence, KV group)
  int items;   // B * nkv * pairs
  int Lq;
  float scale_log2;  // softmax scale * log2(e)
  __half* o;
  unsigned* err;
  // split key ranges: pairs 0 .. nsplit-1 (the longest) run as two halves on any CTAs; each half
  // leaves its unnormalised O, max and sum in part, and the second to finish merges them
  int nsplit;
  int* split_cnt;  // [nsplit][2 tiles][8 softmax warps], zero at launch
  float* part;     // [nsplit][2 halves][2 tiles][PART_TILE]
  // optional: base-2 log-sum-exp of every row's scaled scores, lse2[(b * nq + h) * lse_stride + t]
  float* lse2;
  int lse_stride;
};

// Per-CTA work lists: CTA c runs items[off[c] .. off[c+1]). An entry is a pair index in its low 12
// bits and, in bits 12-13, 0 for the whole key range or 1 / 2 for its first / second half.
struct AttnSched {
  int use;  // 0: serpentine order instead
  unsigned short off[MAX_CTAS + 1];
  unsigned short items[MAX_LIST];
};
constexpr int kEntryPairBits = 12;

struct Item {
  int b, g, nkv_tiles;
  int k0, k1;  // key tiles [k0, k1) of this entry
  int half;    // 0 whole range, 1 / 2 first / second half of a split pair
  int w;       // pair index
  int h[2], qt[2];
  bool active[2];
};

// `entry`: pair index in bits [0, 24), half (0, 1, 2) above.
__device__ __forceinline__ Item get_item(const AttnParams& p, int entry) {
  const int w = entry & 0xffffff;
  const int bgc = p.B * p.nkv;
  const int pr = p.pairs - 1 - w / bgc;  // longest pairs first
  const int bg = w % bgc;
  Item it;
  it.b = bg / p.nkv;
  it.g = bg % p.nkv;
  const int U = p.num_qt * p.G;  // (query tile, head) units of this group, tile-major
  it.nkv_tiles = 0;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int u = 2 * pr + j;
    it.active[j] = u < U;
    const int uu = it.active[j] ? u : 2 * pr;
    it.qt[j] = uu / p.G;
    it.h[j] = it.g * p.G + uu % p.G;
    if (it.active[j] && it.qt[j] + 1 > it.nkv_tiles) it.nkv_tiles = it.qt[j] + 1;
  }
  it.w = w;
  it.half = entry >> 24;
  const int hsplit = it.nkv_tiles / 2;  // split pairs have at least 4 key tiles
  it.k0 = it.half == 2 ? hsplit : 0;
  it.k1 = it.half == 1 ? hsplit : it.nkv_tiles;
  return it;
}

// Work item of this CTA in round r (pair index | half << 24), or -1 when it has none left.
__device__ __forceinline__ int item_index(const AttnSched& sc, int items, int r, int cta, int grid) {
  if (sc.use) {
    const int i = sc.off[cta] + r;
    if (i >= sc.off[cta + 1]) return -1;
    const int e = sc.items[i];
    return (e & ((1 << kEntryPairBits) - 1)) | ((e >> kEntryPairBits) << 24);
  }
  const int w = r * grid + ((r & 1) ? (grid - 1 - cta) : cta);  // serpentine over the CTAs
  return w < items ? w : -1;
}

__global__ void __launch_bounds__(NUM_THREADS, 1) attn_tc_kernel(const __grid_constant__ AttnMaps maps,
                                                                 const AttnParams p,
                                                                 const __grid_constant__ AttnSched sched) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;             // [K_STAGES]
  uint64_t* k_empty = k_full + K_STAGES;   // [K_STAGES]
  uint64_t* v_full = k_empty + K_STAGES;   // [V_STAGES]
  uint64_t* v_empty = v_full + V_STAGES;   // [V_STAGES]
  uint64_t* s_full = v_empty + V_STAGES;   // [2]
  uint64_t* p_full = s_full + 2;           // [2]
  uint64_t* o_full = p_full + 2;           // [2]
  uint64_t* q_stage_free = o_full + 2;     // [2] Q_j's buffer, used to stage O_j, may take the next Q_j
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_stage_free + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    mbar_init(smem_u32(q_empty), 1);
    for (int s = 0; s < K_STAGES; ++s) {
      mbar_init(smem_u32(&k_full[s]), 1);
      mbar_init(smem_u32(&k_empty[s]), 1);
    }
    for (int s = 0; s < V_STAGES; ++s) {
      mbar_init(smem_u32(&v_full[s]), 1);
      mbar_init(smem_u32(&v_empty[s]), 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(smem_u32(&s_full[j]), 1);
      mbar_init(smem_u32(&p_full[j]), 8);
      mbar_init(smem_u32(&o_full[j]), 1);
      mbar_init(smem_u32(&q_stage_free[j]), 8);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.q);
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
  const int cta = blockIdx.x, grid = gridDim.x;

  if (warp == 0) {
    {
      // ------------------------------------------------------------ TMA --
      // Every lane runs this loop and its bounded waits; an elected lane issues each copy.
      int kst = 0, vst = 0;
      uint32_t kph = 0, vph = 0;
      for (int r = 0;; ++r) {
        const int w = item_index(sched, p.items, r, cta, grid);
        if (w < 0) break;
        const Item it = get_item(p, w);
        if (!mbar_wait_bounded(smem_u32(q_empty), (r & 1) ^ 1, p.err, abort_flag, wait_site(kSiteAttn, 1, 1))) goto done;
        // the softmax groups stage the previous entry's O in the Q buffers and release them per tile
        for (int j = 0; j < 2; ++j)
          if (r > 0 && !mbar_wait_bounded(smem_u32(&q_stage_free[j]), (r - 1) & 1, p.err, abort_flag,
                                          wait_site(kSiteAttn, 1, 13)))
            goto done;
        if (elect_one_sync()) mbar_arrive_expect_tx(smem_u32(q_full), 2 * TILE_BYTES);
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            if (elect_one_sync()) tma_load_3d(smem_u32(smem + OFF_Q + j * TILE_BYTES + hf * HALF_BYTES), &maps.q, smem_u32(q_full),
                        it.h[j] * D + hf * 64, it.qt[j] * TQ, it.b);
        // K runs one tile ahead of V: the MMA thread needs K_{jj+1} right after its PVs on V_jj,
        // and a wait for a free V slot must not hold back the next K load
        auto load_k = [&](int jj) -> bool {
          if (!mbar_wait_bounded(smem_u32(&k_empty[kst]), kph ^ 1, p.err, abort_flag, wait_site(kSiteAttn, 1, 2)))
            return false;
          if (elect_one_sync()) mbar_arrive_expect_tx(smem_u32(&k_full[kst]), TILE_BYTES);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            if (elect_one_sync()) tma_load_3d(smem_u32(smem + OFF_K + kst * TILE_BYTES + hf * HALF_BYTES), &maps.k, smem_u32(&k_full[kst]),
                        it.g * D + hf * 64, jj * TK, it.b);
          if (++kst == K_STAGES) {
            kst = 0;
            kph ^= 1;
          }
          return true;
        };
        if (!load_k(it.k0)) goto done;
        for (int jj = it.k0; jj < it.k1; ++jj) {
          if (jj + 1 < it.k1 && !load_k(jj + 1)) goto done;
          if (!mbar_wait_bounded(smem_u32(&v_empty[vst]), vph ^ 1, p.err, abort_flag, wait_site(kSiteAttn, 1, 3))) goto done;
          if (elect_one_sync()) mbar_arrive_expect_tx(smem_u32(&v_full[vst]), TILE_BYTES);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            if (elect_one_sync()) tma_load_3d(smem_u32(smem + OFF_V + vst * TILE_BYTES + hf * HALF_BYTES), &maps.v, smem_u32(&v_full[vst]),
                        it.g * D + hf * 64, jj * TK, it.b);
          if (++vst == V_STAGES) {
            vst = 0;
            vph ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    {
      // ------------------------------------------------------------ MMA --
      // Every lane runs this loop and its bounded waits; elect_one_sync picks the lane that issues
      // each tcgen05 instruction (issuing from a lane-divergent branch costs more per MMA).
      const uint32_t idesc_qk = idesc_f32acc(TQ, TK, 0, 0, kFmtF16);  // Q, K both K-major (d contiguous)
      const uint32_t idesc_pv = idesc_f32acc(TQ, D, 0, 1, kFmtF16);   // P from TMEM, V MN-major (d contiguous)
      int kst = 0, vst = 0;
      uint32_t kph = 0, vph = 0;
      uint32_t pcount[2] = {0, 0};
      // K-major tiles (Q, K): LBO unused, SBO = 1024 B between 8-row groups; V (MN-major): LBO =
      // HALF_BYTES between the two 64-column halves of d, SBO = 1024 B between 8-key groups.
      // The start-address field counts 16-byte units, so stepping a tile by TILE_BYTES adds TILE_BYTES / 16.
      const uint32_t sw_hi = desc_hi(smem_desc_sw128(smem_u32(smem), 16, 1024));
      const uint32_t v_hi = desc_hi(smem_desc_sw128(smem_u32(smem), HALF_BYTES, 1024));
      const uint32_t q_lo0 = desc_lo(smem_desc_sw128(smem_u32(smem + OFF_Q), 16, 1024));
      const uint32_t k_lo0 = desc_lo(smem_desc_sw128(smem_u32(smem + OFF_K), 16, 1024));
      const uint32_t v_lo0 = desc_lo(smem_desc_sw128(smem_u32(smem + OFF_V), HALF_BYTES, 1024));
      constexpr uint32_t kTileStep = TILE_BYTES >> 4;
      for (int r = 0;; ++r) {
        const int w = item_index(sched, p.items, r, cta, grid);
        if (w < 0) break;
        const Item it = get_item(p, w);
        if (!mbar_wait_bounded(smem_u32(q_full), r & 1, p.err, abort_flag, wait_site(kSiteAttn, 2, 4))) goto done;
        // O_j of the previous pair needs no guard: the first PV of this pair waits for p_full[j],
        // which the softmax group raises only after its epilogue has read O_j back.
        tc_fence_after();
        // S_j = Q_j K_st^T: descriptors built once, the K = 16 steps advance the start address
        // (16-byte units) by 2 within a 128-byte row and by HALF_BYTES / 16 per d half
        auto issue_qk = [&](int j, int st) {
          const uint32_t alo = q_lo0 + j * kTileStep, blo = k_lo0 + st * kTileStep;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4;
            if (elect_one_sync()) umma_ss_lohi(tmem + COL_S0 + j * TK, alo + off, sw_hi, blo + off, sw_hi, idesc_qk, kk > 0);
          }
          if (elect_one_sync()) umma_commit(smem_u32(&s_full[j]));
        };
        // first key tile: S_j = Q_j K_0^T for both tiles
        if (!mbar_wait_bounded(smem_u32(&k_full[kst]), kph, p.err, abort_flag, wait_site(kSiteAttn, 2, 6))) goto done;
        tc_fence_after();
        for (int j = 0; j < 2; ++j)
          if (it.active[j]) issue_qk(j, kst);
        if (elect_one_sync()) umma_commit(smem_u32(&k_empty[kst]));
        if (++kst == K_STAGES) {
          kst = 0;
          kph ^= 1;
        }
        for (int jj = it.k0; jj < it.k1; ++jj) {
          bool next_k_ready = false;
          if (!mbar_wait_bounded(smem_u32(&v_full[vst]), vph, p.err, abort_flag, wait_site(kSiteAttn, 2, 7))) goto done;
          tc_fence_after();
          const uint32_t vlo = v_lo0 + vst * kTileStep;
          for (int j = 0; j < 2; ++j) {
            if (!it.active[j] || jj > it.qt[j]) continue;
            if (!mbar_wait_bounded(smem_u32(&p_full[j]), pcount[j] & 1, p.err, abort_flag, wait_site(kSiteAttn, 2, 8))) goto done;
            ++pcount[j];
            tc_fence_after();
            // O_j += P_j V_jj
#pragma unroll
            for (int kk = 0; kk < TK / 16; ++kk)
              if (elect_one_sync()) umma_ts_lohi(tmem + COL_O0 + j * D, tmem + COL_S0 + j * TK + kk * 8, vlo + ((kk * 16 * 128) >> 4),
                           v_hi, idesc_pv, (jj > it.k0 || kk > 0));
            if (jj + 1 <= it.qt[j] && jj + 1 < it.k1) {
              if (!next_k_ready) {
                if (!mbar_wait_bounded(smem_u32(&k_full[kst]), kph, p.err, abort_flag, wait_site(kSiteAttn, 2, 9))) goto done;
                tc_fence_after();
                next_k_ready = true;
              }
              issue_qk(j, kst);  // S_j = Q_j K_{jj+1}^T, overwrites P_j after the PV above
            } else {
              if (elect_one_sync()) umma_commit(smem_u32(&o_full[j]));
            }
          }
          if (elect_one_sync()) umma_commit(smem_u32(&v_empty[vst]));
          if (++vst == V_STAGES) {
            vst = 0;
            vph ^= 1;
          }
          if (next_k_ready) {
            if (elect_one_sync()) umma_commit(smem_u32(&k_empty[kst]));
            if (++kst == K_STAGES) {
              kst = 0;
              kph ^= 1;
            }
          }
        }
        if (elect_one_sync()) umma_commit(smem_u32(q_empty));
      }
    }
  } else {
    // -------------------------------------------------------- softmax --
    // Eight warps per tile, two on each SMSP: warp (quad, hf) owns the 16 rows 32 quad + 16 hf .. +15
    // of its TMEM lane quadrant. With the 16-lane TMEM shapes thread t holds rows ra = base + t/4 and
    // rb = ra + 8, and of every 8-key chunk c the keys 8c + 2(t%4) + {0, 1}: a row is spread over
    // the four threads of a quad, which combine its max with two shuffles; the row sums stay
    // per thread until the epilogue.
    const int sw = warp - 2;                // 0 .. 15
    const int j = sw >> 3;                  // tile of this warp
    const int wt = sw & 7;                  // warp within the tile
    const int quad = warp & 3;              // TMEM lanes [32*quad, 32*quad + 32)
    const int rbase = quad * 32 + ((wt >> 2) << 4);  // first of this warp's 16 rows
    const int qd = lane & 3;                // key pair within each 8-key chunk
    const int ra = rbase + (lane >> 2), rb = ra + 8;
    const uint32_t lane_off = (uint32_t)rbase << 16;
    const uint32_t s_col = tmem + lane_off + COL_S0 + j * TK;
    const uint32_t o_col = tmem + lane_off + COL_O0 + j * D;
    uint32_t scount = 0, ocount = 0;
    for (int r = 0;; ++r) {
      const int w = item_index(sched, p.items, r, cta, grid);
      if (w < 0) break;
      const Item it = get_item(p, w);
      if (it.active[j]) {
        const int qt = it.qt[j];
        float ma = -INFINITY, mb = -INFINITY;  // running max of scaled scores (log2 domain), rows ra / rb
        float la = 0.f, lb = 0.f;              // this thread's share of the running row sums
        const int jlast = qt < it.k1 - 1 ? qt : it.k1 - 1;  // last key tile of this entry for the tile
        for (int jj = it.k0; jj <= jlast; ++jj) {
          if (!mbar_wait_bounded(smem_u32(&s_full[j]), scount & 1, p.err, abort_flag, wait_site(kSiteAttn, 3, 10))) goto done;
          ++scount;
          tc_fence_after();
          uint32_t s[64];  // s[4c + e]: row ra, key 8c + 2qd + e; s[4c + 2 + e]: row rb (c = 0 .. 15)
          tmem_ld_16x256b_x8(s_col, s);
          tmem_ld_16x256b_x8(s_col + 64, s + 32);
          tmem_ld_wait();
          if (jj == qt) {  // diagonal tile: key c is visible to query row iff c <= row
#pragma unroll
            for (int c = 0; c < 16; ++c)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int key = 8 * c + 2 * qd + e;
                if (key > ra) s[4 * c + e] = __float_as_uint(-INFINITY);
                if (key > rb) s[4 * c + 2 + e] = __float_as_uint(-INFINITY);
              }
          }
          // row max of the raw scores (the scale is positive): two chains per row, then the quad
          float xa0 = -INFINITY, xa1 = -INFINITY, xb0 = -INFINITY, xb1 = -INFINITY;
#pragma unroll
          for (int c = 0; c < 16; c += 2) {
            xa0 = max3f(xa0, u2f(s[4 * c + 0]), u2f(s[4 * c + 1]));
            xb0 = max3f(xb0, u2f(s[4 * c + 2]), u2f(s[4 * c + 3]));
            xa1 = max3f(xa1, u2f(s[4 * c + 4]), u2f(s[4 * c + 5]));
            xb1 = max3f(xb1, u2f(s[4 * c + 6]), u2f(s[4 * c + 7]));
          }
          float ta = fmaxf(xa0, xa1), tb = fmaxf(xb0, xb1);
          ta = fmaxf(ta, __shfl_xor_sync(0xffffffffu, ta, 1));
          tb = fmaxf(tb, __shfl_xor_sync(0xffffffffu, tb, 1));
          ta = fmaxf(ta, __shfl_xor_sync(0xffffffffu, ta, 2)) * p.scale_log2;
          tb = fmaxf(tb, __shfl_xor_sync(0xffffffffu, tb, 2)) * p.scale_log2;
          // lazy rescale: keep the stale max unless it grew by more than 2^8
          float fa = 1.f, fb = 1.f;  // factors for the O rows and the sums
          if (jj == it.k0) {
            ma = ta;
            mb = tb;
          } else if (__any_sync(0xffffffffu, ta > ma + RESCALE_THRESHOLD || tb > mb + RESCALE_THRESHOLD)) {
            const float na = fmaxf(ma, ta), nb = fmaxf(mb, tb);
            fa = fast_exp2(ma - na);
            fb = fast_exp2(mb - nb);
            ma = na;
            mb = nb;
            // O_j is stable: the commit behind s_full covered the previous PV, and this warp raises
            // p_full (which lets the next PV in) only after these stores have completed
#pragma unroll 1
            for (int g = 0; g < 4; ++g) {
              uint32_t o[16];
              tmem_ld_16x256b_x4(o_col + g * 32, o);
              tmem_ld_wait();
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                o[4 * c + 0] = __float_as_uint(u2f(o[4 * c + 0]) * fa);
                o[4 * c + 1] = __float_as_uint(u2f(o[4 * c + 1]) * fa);
                o[4 * c + 2] = __float_as_uint(u2f(o[4 * c + 2]) * fb);
                o[4 * c + 3] = __float_as_uint(u2f(o[4 * c + 3]) * fb);
              }
              tmem_st_16x256b_x4(o_col + g * 32, o);
            }
          }
          const float sc = p.scale_log2, nma = -ma, nmb = -mb;
          float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;  // packed partial row sums
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            // P columns 32 h2 .. 32 h2 + 31 (keys 64 h2 .. 64 h2 + 63) over the first half of S_j:
            // pk[2cc] = row ra, pk[2cc + 1] = row rb, column 32 h2 + 4 cc + qd (keys 8c + 2qd, +1)
            uint32_t pk[16];
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
              const int c = 8 * h2 + cc;
              float x0, x1, x2, x3, p0, p1, p2, p3;
              fma2(x0, x1, u2f(s[4 * c + 0]), u2f(s[4 * c + 1]), sc, sc, nma, nma);
              fma2(x2, x3, u2f(s[4 * c + 2]), u2f(s[4 * c + 3]), sc, sc, nmb, nmb);
              if (CCA_POLY_EVERY > 0 && (cc % (CCA_POLY_EVERY > 0 ? CCA_POLY_EVERY : 1)) == CCA_POLY_EVERY - 1) {
                exp2_fma_x2(x0, x1, p0, p1);
                exp2_fma_x2(x2, x3, p2, p3);
              } else {
                p0 = fast_exp2(x0);
                p1 = fast_exp2(x1);
                p2 = fast_exp2(x2);
                p3 = fast_exp2(x3);
              }
              add2(sa0, sa1, sa0, sa1, p0, p1);
              add2(sb0, sb1, sb0, sb1, p2, p3);
              pk[2 * cc] = pack_f16x2(p0, p1);
              pk[2 * cc + 1] = pack_f16x2(p2, p3);
            }
            tmem_st_16x128b_x8(s_col + h2 * 32, pk);
          }
          la = la * fa + (sa0 + sa1);
          lb = lb * fb + (sb0 + sb1);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&p_full[j]));
        }
        // epilogue: O / l -> fp16 -> global
        la += __shfl_xor_sync(0xffffffffu, la, 1);
        lb += __shfl_xor_sync(0xffffffffu, lb, 1);
        la += __shfl_xor_sync(0xffffffffu, la, 2);
        lb += __shfl_xor_sync(0xffffffffu, lb, 2);
        // the rows' log-sum-exp (a half of a split pair leaves it to the merge below): the sums are
        // relative to the running max, so lse2 = max + log2(sum)
        float* lse_row = p.lse2 != nullptr ? p.lse2 + ((size_t)it.b * p.nq + it.h[j]) * p.lse_stride : nullptr;
        const int ta = qt * TQ + ra, tb = qt * TQ + rb;
        if (lse_row != nullptr && it.half == 0 && qd == 0) {
          if (ta < p.S) lse_row[ta] = ma + log2f(la);
          if (tb < p.S) lse_row[tb] = mb + log2f(lb);
        }
        if (!mbar_wait_bounded(smem_u32(&o_full[j]), ocount & 1, p.err, abort_flag, wait_site(kSiteAttn, 3, 11))) goto done;
        ++ocount;
        tc_fence_after();
        // O_row = O * inv for a whole-range entry; a merged split pair gives c1 * O_first + c2 * O_second,
        // evaluated in that order whichever half merges, so the result does not depend on timing
        float c1a = 0.f, c2a = 0.f, c1b = 0.f, c2b = 0.f, inva = 1.f / la, invb = 1.f / lb;
        const float* other = nullptr;
        bool store = true;
        if (it.half != 0) {
          // one half of a split pair: publish this half's unnormalised rows with their max and sum
          // ([16 chunks of 8 columns][128 rows][8] fp32, then max [128] and sum [128]); the second of
          // the two halves to get here (counted per warp) merges them
          const size_t tile = (size_t)it.w * 2 + j;
          float* mine = p.part + ((size_t)it.w * 4 + (it.half - 1) * 2 + j) * PART_TILE;
          other = p.part + ((size_t)it.w * 4 + (2 - it.half) * 2 + j) * PART_TILE;
#pragma unroll 1
          for (int g = 0; g < 4; ++g) {
            uint32_t o[16];
            tmem_ld_16x256b_x4(o_col + g * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int ch = 4 * g + c;
              *reinterpret_cast<float2*>(mine + ((size_t)ch * TQ + ra) * 8 + 2 * qd) =
                  make_float2(u2f(o[4 * c + 0]), u2f(o[4 * c + 1]));
              *reinterpret_cast<float2*>(mine + ((size_t)ch * TQ + rb) * 8 + 2 * qd) =
                  make_float2(u2f(o[4 * c + 2]), u2f(o[4 * c + 3]));
            }
          }
          if (qd == 0) {
            mine[D * TQ + ra] = ma;
            mine[D * TQ + rb] = mb;
            mine[D * TQ + TQ + ra] = la;
            mine[D * TQ + TQ + rb] = lb;
          }
          __threadfence();
          __syncwarp();
          int ticket = 0;
          if (lane == 0) ticket = atomicAdd(p.split_cnt + tile * 8 + wt, 1);
          ticket = __shfl_sync(0xffffffffu, ticket, 0);
          store = ticket != 0;
          if (store) {
            __threadfence();
            const bool first = it.half == 1;  // this half holds O_first
            auto coeffs = [&](int row, float m, float l, float& c1, float& c2, float& lse) {
              const float mo = __ldcg(other + D * TQ + row), lo = __ldcg(other + D * TQ + TQ + row);
              const float m1 = first ? m : mo, l1 = first ? l : lo;
              const float m2 = first ? mo : m, l2 = first ? lo : l;
              const float mm = fmaxf(m1, m2);
              const float e1 = fast_exp2(m1 - mm), e2 = fast_exp2(m2 - mm);
              const float lsum = __fmaf_rn(e1, l1, __fmul_rn(e2, l2));
              const float rl = 1.f / lsum;
              c1 = __fmul_rn(e1, rl);
              c2 = __fmul_rn(e2, rl);
              lse = mm + log2f(lsum);
            };
            float lsea, lseb;
            coeffs(ra, ma, la, c1a, c2a, lsea);
            coeffs(rb, mb, lb, c1b, c2b, lseb);
            if (lse_row != nullptr && qd == 0) {
              if (ta < p.S) lse_row[ta] = lsea;
              if (tb < p.S) lse_row[tb] = lseb;
            }
            inva = invb = 1.f;  // the raw O rows are merged
          }
        }
        // O rows leave through Q_j's buffer (its last QK has completed): [2 halves][128 rows][128 B]
        // with the 128-byte swizzle, one TMA tensor store per 64-column half of this warp's 16 rows
        uint8_t* stage = smem + OFF_Q + j * TILE_BYTES;
#pragma unroll 1
        for (int g = 0; g < 4 && store; ++g) {
          uint32_t o[16];
          tmem_ld_16x256b_x4(o_col + g * 32, o);
          tmem_ld_wait();
          float f[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            f[4 * c + 0] = u2f(o[4 * c + 0]) * inva;
            f[4 * c + 1] = u2f(o[4 * c + 1]) * inva;
            f[4 * c + 2] = u2f(o[4 * c + 2]) * invb;
            f[4 * c + 3] = u2f(o[4 * c + 3]) * invb;
          }
          if (other != nullptr) {
            const bool first = it.half == 1;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int ch = 4 * g + c;
              const float2 xa = __ldcg(reinterpret_cast<const float2*>(other + ((size_t)ch * TQ + ra) * 8 + 2 * qd));
              const float2 xb = __ldcg(reinterpret_cast<const float2*>(other + ((size_t)ch * TQ + rb) * 8 + 2 * qd));
              const float x[4] = {xa.x, xa.y, xb.x, xb.y};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float k1 = u < 2 ? c1a : c1b, k2 = u < 2 ? c2a : c2b;
                const float o1 = first ? f[4 * c + u] : x[u], o2 = first ? x[u] : f[4 * c + u];
                f[4 * c + u] = __fmaf_rn(k1, o1, __fmul_rn(k2, o2));
              }
            }
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {  // columns 8 ch + 2 qd, +1 of 16-byte chunk ch: half ch / 8, chunk ch % 8
            const int ch = 4 * g + c;
            uint8_t* base = stage + (ch >> 3) * HALF_BYTES + 4 * qd;
            *reinterpret_cast<uint32_t*>(base + ra * 128 + (((ch & 7) ^ (ra & 7)) << 4)) =
                pack_f16x2(f[4 * c + 0], f[4 * c + 1]);
            *reinterpret_cast<uint32_t*>(base + rb * 128 + (((ch & 7) ^ (rb & 7)) << 4)) =
                pack_f16x2(f[4 * c + 2], f[4 * c + 3]);
          }
        }
        if (store) {
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {  // rows past S are clipped by the map
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
              tma_store_3d(&maps.o, smem_u32(stage + hf * HALF_BYTES + rbase * 128), it.h[j] * D + hf * 64,
                           qt * TQ + rbase, it.b);
            bulk_commit();
          }
        }
        tc_fence_before();
      }
      // every entry, active tile or not: Q_j's buffer may take the next entry's Q once this warp's
      // stores have read it
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&q_stage_free[j]));
    }
  }
done:
  if (warp >= 2 && lane == 0) bulk_wait_all();  // staged stores finish before the CTA's shared memory goes
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

bool encode_3d(CUtensorMap* m, const void* ptr, uint64_t width, uint64_t S, uint64_t B, uint32_t box_rows = 128) {
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

// Schedule cost model, in units of about half a key-tile step (one step: both query tiles of the
// pair against one key tile): two per step plus a fixed cost per entry for its setup, pipeline
// fill and epilogue; a half of a split pair pays more for publishing or merging its partial rows.
// The constants follow per-entry timings of this kernel on B200 (about 2 us per step, 4 to 6 us
// per entry, 4 us more for a split half); nkv = key tiles of the pair.
struct PairGeom {
  int num_qt, pairs, items, bgc, U;
  explicit PairGeom(const BlockDims& dm)
      : num_qt((dm.S + TQ - 1) / TQ),
        pairs((num_qt * dm.G + 1) / 2),
        items(dm.B * dm.nkv * pairs),
        bgc(dm.B * dm.nkv),
        U(num_qt * dm.G) {}
  int nkv(const BlockDims& dm, int w) const {
    const int pr = pairs - 1 - w / bgc;
    return (2 * pr + 1 < U ? 2 * pr + 1 : 2 * pr) / dm.G + 1;
  }
  static constexpr int kEntryCost = 4, kSplitCost = 4;
  int load(const BlockDims& dm, int w) const { return 2 * nkv(dm, w) + kEntryCost; }
  // Most pairs that may be split in two (the longest ones, with at least 4 key tiles so that both
  // query tiles have keys in both halves).
  int max_split(const BlockDims& dm) const {
    if (items > MAX_LIST) return 0;
    int n = 0;
    while (n < items && n < kAttnMaxSplit && n + items < MAX_LIST && nkv(dm, n) >= 4) ++n;
    return n;
  }
};

// Entries for the first ns pairs split in two, in non-increasing order of cost. Returns the count.
int build_entries(const BlockDims& dm, const PairGeom& g, int ns, unsigned short* entry, int* cost) {
  unsigned short he[2 * kAttnMaxSplit];
  int hc[2 * kAttnMaxSplit], nh = 0;
  for (int w = 0; w < ns; ++w) {
    const int nk = g.nkv(dm, w), h = nk / 2;
    he[nh] = (unsigned short)(w | (2 << kEntryPairBits));
    hc[nh++] = 2 * (nk - h) + PairGeom::kEntryCost + PairGeom::kSplitCost;
    he[nh] = (unsigned short)(w | (1 << kEntryPairBits));
    hc[nh++] = 2 * h + PairGeom::kEntryCost + PairGeom::kSplitCost;
  }
  for (int i = 1; i < nh; ++i)  // insertion sort, non-increasing (stable)
    for (int k = i; k > 0 && hc[k - 1] < hc[k]; --k) {
      const int c = hc[k];
      hc[k] = hc[k - 1];
      hc[k - 1] = c;
      const unsigned short e = he[k];
      he[k] = he[k - 1];
      he[k - 1] = e;
    }
  int n = 0, i = 0, w = ns;  // merge with the whole pairs ns .. items-1 (already non-increasing)
  while (i < nh || w < g.items) {
    if (w >= g.items || (i < nh && hc[i] >= g.load(dm, w))) {
      entry[n] = he[i];
      cost[n++] = hc[i++];
    } else {
      entry[n] = (unsigned short)w;
      cost[n++] = g.load(dm, w++);
    }
  }
  return n;
}

// Longest-processing-time assignment of entries (in order) to `grid` CTAs, each to the CTA with the
// least work so far (a binary min-heap of CTA loads). Fills owner[] and count[]; returns the largest
// CTA load.
long long assign_lpt(int n, const int* cost, int grid, unsigned short* owner, int* count) {
  long long load[MAX_CTAS];
  int heap_cta[MAX_CTAS];
  for (int c = 0; c < grid; ++c) {
    load[c] = 0;
    heap_cta[c] = c;
    count[c] = 0;
  }
  auto less = [&](int a, int b) { return load[a] < load[b] || (load[a] == load[b] && a < b); };
  for (int i = 0; i < n; ++i) {
    const int c = heap_cta[0];
    owner[i] = (unsigned short)c;
    ++count[c];
    load[c] += cost[i];
    for (int x = 0;;) {  // sift the root down
      const int l = 2 * x + 1, r = l + 1;
      int m = x;
      if (l < grid && less(heap_cta[l], heap_cta[m])) m = l;
      if (r < grid && less(heap_cta[r], heap_cta[m])) m = r;
      if (m == x) break;
      const int t = heap_cta[x];
      heap_cta[x] = heap_cta[m];
      heap_cta[m] = t;
      x = m;
    }
  }
  long long mx = 0;
  for (int c = 0; c < grid; ++c) mx = load[c] > mx ? load[c] : mx;
  return mx;
}

constexpr size_t kCounterBytes = (size_t)kAttnSplitCounters * sizeof(int);
constexpr size_t kPartSlotBytes = (size_t)2 * 2 * PART_TILE * sizeof(float);

}  // namespace

size_t attention_tc_scratch_bytes(const BlockDims& dm) {
  // the largest split set of any grid (at most MAX_CTAS CTAs)
  return kCounterBytes + (size_t)PairGeom(dm).max_split(dm) * kPartSlotBytes;
}

bool attention_tc_supported(const BlockDims& dm) {
  return dm.lat == DType::F16 && dm.d == D && dm.S >= 1 && (long long)dm.Lq * dm.S * 2 < (1ll << 40);
}

cudaError_t launch_attention_tc(const BlockDims& dm, const void* q, const void* k, const void* v, void* o,
                                void* scratch, unsigned* dev_err, cudaStream_t stream, float* lse2, int lse_stride) {
  if (!attention_tc_supported(dm)) return cudaErrorInvalidValue;
  AttnMaps maps;
  if (!encode_3d(&maps.q, q, (uint64_t)dm.Lq, (uint64_t)dm.S, (uint64_t)dm.B) ||
      !encode_3d(&maps.k, k, (uint64_t)dm.Lkv, (uint64_t)dm.S, (uint64_t)dm.B) ||
      !encode_3d(&maps.v, v, (uint64_t)dm.Lkv, (uint64_t)dm.S, (uint64_t)dm.B) ||
      !encode_3d(&maps.o, o, (uint64_t)dm.Lq, (uint64_t)dm.S, (uint64_t)dm.B, 16))
    return cudaErrorInvalidValue;
  AttnParams p;
  p.B = dm.B;
  p.S = dm.S;
  p.nq = dm.nq;
  p.nkv = dm.nkv;
  p.G = dm.G;
  p.num_qt = (dm.S + TQ - 1) / TQ;
  p.pairs = (p.num_qt * dm.G + 1) / 2;
  p.items = dm.B * dm.nkv * p.pairs;
  p.Lq = dm.Lq;
  p.scale_log2 = dm.scale * 1.4426950408889634f;
  p.o = static_cast<__half*>(o);
  p.err = dev_err;
  p.lse2 = lse2;
  p.lse_stride = lse_stride;
  int grid = p.items < num_sms() ? p.items : num_sms();
  if (grid > MAX_CTAS) grid = MAX_CTAS;
  p.split_cnt = static_cast<int*>(scratch);
  p.part = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + kCounterBytes);
  // Schedule: the longest pairs may run as two halves of their key range (merged by the half that
  // ends second); of all split counts the one with the smallest simulated makespan is taken. The
  // plan depends on the shape and the grid only and is kept for the next launch of the same shape.
  // Fixed-size arrays only: launching allocates no memory.
  struct PlanCache {
    int key[6] = {-1, -1, -1, -1, -1, -1};
    int nsplit = 0;
    AttnSched plan;
  };
  static thread_local PlanCache cache;
  const int key[6] = {dm.B, dm.S, dm.G, dm.nkv, grid, (int)PairGeom(dm).items};
  bool hit = true;
  for (int i = 0; i < 6; ++i) hit = hit && cache.key[i] == key[i];
  if (!hit) {
    const PairGeom geom(dm);
    static thread_local unsigned short owner[MAX_LIST], entry[MAX_LIST];
    static thread_local int cost[MAX_LIST];
    int count[MAX_CTAS];
    AttnSched& plan = cache.plan;
    plan.use = p.items <= MAX_LIST;
    cache.nsplit = 0;
    if (plan.use) {
      long long best = -1;
      const int maxs = geom.max_split(dm);
      for (int ns = 0; ns <= maxs; ++ns) {
        const int n = build_entries(dm, geom, ns, entry, cost);
        const long long mk = assign_lpt(n, cost, grid, owner, count);
        if (best < 0 || mk < best) {
          best = mk;
          cache.nsplit = ns;
        }
      }
      const int n = build_entries(dm, geom, cache.nsplit, entry, cost);
      assign_lpt(n, cost, grid, owner, count);
      int off = 0;
      for (int c = 0; c < grid; ++c) {
        plan.off[c] = (unsigned short)off;
        off += count[c];
        count[c] = plan.off[c];  // fill cursor
      }
      plan.off[grid] = (unsigned short)off;
      for (int i = 0; i < n; ++i) plan.items[count[owner[i]]++] = entry[i];
    }
    for (int i = 0; i < 6; ++i) cache.key[i] = key[i];
  }
  p.nsplit = cache.nsplit;
  const AttnSched& plan = cache.plan;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(maps, p, plan);
  return cudaGetLastError();
}

}  // namespace cca
