// Tensor-core GEMM for sm_100a: C[M, N] = A[M, K] * B[N, K]^T, 16-bit inputs
// (bf16 or fp16), fp32 accumulation in tensor memory, fp32 / bf16 / fp16
// output.
//
// Used for the two dense projections of a CCA block ("Compressed
// Convolutional Attention", gist.science/es/paper/2510.04476, section 2.A):
// the down-projection of the hidden states to the q~ | k~ | v~ latents (the B
// operand is W_q, W_k, W_v stacked by rows, each in its own buffer) and the
// output projection o W_o^T.
//
// Design: persistent CTAs (one per SM) walk 128 x 256 output tiles. Warp 0
// issues TMA loads of 128 x 64 A tiles and 256 x 64 B tiles (128-byte swizzle)
// into a 4-stage shared-memory ring; warp 1 runs the MMA loop and an elected
// lane issues tcgen05.mma (M=128, N=256, K=16) into one of two 256-column fp32
// accumulators in tensor memory; warps 2-5 drain the other accumulator so the
// epilogue of tile i overlaps the main loop of tile i+1. For 16-bit outputs
// each epilogue warp converts 32 rows x 64 columns at a time into its own
// staging buffer (128-byte swizzle) and one of its threads writes the chunk
// with a TMA tensor store, so global writes leave in whole lines; fp32
// outputs are stored directly. Every mbarrier wait is bounded.
//
// GEMMs of at least 256 rows use the pair form (clusters of two CTAs, tcgen05
// cta_group::2) with 256 x 256 tiles: each CTA loads 128 rows of A and 128
// rows of B per K step, the even CTA issues M=256 MMAs that read both CTAs'
// shared memory, and each CTA drains its 128 rows from its own tensor memory,
// still double-buffered. Per FLOP a CTA loads two thirds of what a 128 x 256
// tile needs. The single-CTA forms (128 x 256, and 256 x 256 with one
// accumulator pair for long K) serve smaller M, or a device where a cluster
// of two of these CTAs does not fit.
#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

constexpr int BN = 256, BK = 64;
constexpr int A_HALF_BYTES = 128 * BK * 2;  // 128 rows of A, 16 KB
constexpr int MN_CHUNK_BYTES = 64 * BK * 2;  // an MN-major operand's [64 K][64 M or N] chunk, 8 KB
constexpr int TMEM_COLS = 512;

// Two tile shapes. MH = 1: 128 x 256 tiles, 4 stages of 48 KB, two 256-column accumulators so the
// epilogue of one tile overlaps the main loop of the next. MH = 2: 256 x 256 tiles (two 128-row
// MMAs per K step share the B tile, so the operands cross from L2 a third less often per flop),
// 3 stages of 64 KB, one accumulator pair filling all 512 columns, eight epilogue warps.
// PAIR: tiles of 256 * MH rows x 256 columns split over a cluster of two CTAs: each CTA holds MH
// 128-row blocks of A (block h of CTA r is tile rows h*256 + r*128 ..) and 128 of the B rows;
// MH = 1 takes 6 stages of 32 KB, MH = 2 4 stages of 48 KB. Only MH = 1 pairs are launched: 256
// rows per CTA (one accumulator pair, no epilogue overlap) measured no faster.
template <int MH, bool PAIR = false>
struct Shape {
  static constexpr int BM = 128 * MH;  // rows of this CTA's share of a tile
  static constexpr int TM = BM * (PAIR ? 2 : 1);  // rows of a tile
  static constexpr int HS = PAIR ? 256 : 128;     // tile rows between this CTA's 128-row blocks
  static constexpr int B_ROWS = PAIR ? 128 : BN;  // B rows this CTA loads per K step
  static constexpr int STAGES = PAIR ? (MH == 1 ? 6 : 4) : (MH == 1 ? 4 : 3);
  static constexpr int A_BYTES = A_HALF_BYTES * MH;
  static constexpr int STAGE_BYTES = A_BYTES + B_ROWS * BK * 2;
  static constexpr int ACC_BUFS = MH == 1 ? 2 : 1;
  static constexpr int EPI_WARPS = 4 * MH;
  static constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
  // per epilogue warp, staging buffers of 32 rows x 64 columns (16-bit) for TMA stores (MH = 1)
  static constexpr int EPI_BUFS = MH == 1 ? 2 : 0;
  static constexpr int STG_BYTES = 32 * 64 * 2;
  static constexpr size_t SMEM_BYTES = (size_t)STAGES * STAGE_BYTES + (size_t)EPI_WARPS * EPI_BUFS * STG_BYTES +
                                       1024 /*align slack*/ + 256 /*barriers*/;
  static_assert(SMEM_BYTES <= 232448, "shared memory of one CTA");
  static constexpr int EPI_BUF_COUNT = EPI_BUFS > 0 ? EPI_BUFS : 1;  // (unused when MH = 2)
};

struct GemmMaps {
  CUtensorMap a;
  CUtensorMap b[3];
  CUtensorMap c;  // 16-bit output, boxes of 64 columns x 32 rows (used when tma_store)
};

struct GemmParams {
  long long M;
  int N, K;
  int nb;
  int row_start[3];  // first row of B matrix i in the stacked operand
  int nrows[3];
  void* C;
  long long ldc;
  int out_type;  // DType of C
  int in_fmt;    // kFmtBF16 or kFmtF16
  unsigned* err;
  int num_tiles;  // work items: output tiles x K slices
  int n_tiles_n;
  int tiles;      // output tiles
  int ksplit;     // K slices per tile (fp32 output added with reductions when > 1)
  int kb_slice;   // 64-deep K blocks per slice
  int a_kwrap, b_kwrap;  // the operand's own K extent when it repeats along K (0: K)
  int a_mn, b_mn;        // operand stored [K][M] ([K][N]): loaded as 64 x 64 boxes, read MN-major
  int tma_store;  // 16-bit output written through shared memory and maps.c
  // side job (bf16 -> fp16 copies), done by the epilogue warps before their first tile
  const __nv_bfloat16* side_src[2];
  __half* side_dst[2];
  long long side_n[2];
  float side_scale;
  // value shift in the epilogue (v_cache non-null): see GemmTcArgs
  __nv_bfloat16* v_cache;
  __half* v_att;
  int v_col0, Lkv, S, vshift, vfrom;
};

// The value shift of 64 accumulators of one row of v~ (columns vc .. vc + 63 of the V latent): the bf16
// cache and the fp16 attention copy, one row down within the sequence for the shifted channels
// (nothing past the sequence end; zeros at its start). Returns true if an fp16 value overflowed.
__device__ __forceinline__ bool store_value_shift(const GemmParams& p, long long row, int vc, const uint32_t* r) {
  const bool shifted = p.vshift && vc >= p.vfrom;
  const long long s = row % p.S;
  bool bad = false;
  if (!shifted || s + 1 < p.S) {
    const long long off = (shifted ? row + 1 : row) * p.Lkv + vc;
    uint4* dh = reinterpret_cast<uint4*>(p.v_att + off);
    uint4* db = reinterpret_cast<uint4*>(p.v_cache + off);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      uint32_t h[4], b[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = u2f(r[8 * v + 2 * e]), x1 = u2f(r[8 * v + 2 * e + 1]);
        bad |= f16_overflow(x0) || f16_overflow(x1);
        h[e] = pack_f16x2(x0, x1);
        b[e] = pack_bf16x2(x0, x1);
      }
      dh[v] = make_uint4(h[0], h[1], h[2], h[3]);
      db[v] = make_uint4(b[0], b[1], b[2], b[3]);
    }
  }
  if (shifted && s == 0) {
    const long long off = row * p.Lkv + vc;
    uint4* dh = reinterpret_cast<uint4*>(p.v_att + off);
    uint4* db = reinterpret_cast<uint4*>(p.v_cache + off);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      dh[v] = make_uint4(0, 0, 0, 0);
      db[v] = make_uint4(0, 0, 0, 0);
    }
  }
  return bad;
}

// Stores 32 fp32 accumulators of one row; returns true if an fp16 output overflowed.
__device__ __forceinline__ bool store_row_chunk(const GemmParams& p, long long row, int col0, const uint32_t* r) {
  bool bad = false;
  if (p.out_type == (int)DType::BF16 || p.out_type == (int)DType::F16) {
    const bool h = p.out_type == (int)DType::F16;
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.C) + row * p.ldc + col0);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = u2f(r[8 * v + 2 * e]), b = u2f(r[8 * v + 2 * e + 1]);
        if (h) {
          w[e] = pack_f16x2(a, b);
          bad |= f16_overflow(a) || f16_overflow(b);
        } else {
          w[e] = pack_bf16x2(a, b);
        }
      }
      dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else if (p.ksplit > 1) {  // a K slice's share, added to the sum of all slices
    float* dst = static_cast<float*>(p.C) + row * p.ldc + col0;
#pragma unroll
    for (int v = 0; v < 8; ++v)
      asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + 4 * v), "f"(u2f(r[4 * v])),
                   "f"(u2f(r[4 * v + 1])), "f"(u2f(r[4 * v + 2])), "f"(u2f(r[4 * v + 3]))
                   : "memory");
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(p.C) + row * p.ldc + col0);
#pragma unroll
    for (int v = 0; v < 8; ++v) dst[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
  }
  return bad;
}

// GEN: the general form (K slices, K-wrapped operands, MN-major operands). Without it those
// parameters are compile-time off and the loops are the plain K-major ones: the forward's
// projections are bound by the rate TMA copies and MMAs are issued at, and the general form's
// runtime selections measured 15-20 % slower there.
template <int MH, bool PAIR, bool GEN>
__global__ void __launch_bounds__(Shape<MH, PAIR>::NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
  using T = Shape<MH, PAIR>;
  const bool a_mn = GEN && p.a_mn, b_mn = GEN && p.b_mn;
  const int a_kwrap = GEN ? p.a_kwrap : 0, b_kwrap = GEN ? p.b_kwrap : 0;
  const int tiles = GEN ? p.tiles : p.num_tiles;
  constexpr int BM = T::BM, TM = T::TM, STAGES = T::STAGES, STAGE_BYTES = T::STAGE_BYTES, A_BYTES = T::A_BYTES;
  constexpr int ACC_BUFS = T::ACC_BUFS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + STAGES * STAGE_BYTES;  // [EPI_WARPS][EPI_BUFS][32 rows][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + T::EPI_WARPS * T::EPI_BUFS * T::STG_BYTES);
  uint64_t* full = bars;                 // [STAGES] TMA -> MMA
  uint64_t* empty = bars + STAGES;       // [STAGES] MMA -> TMA
  uint64_t* tfull = bars + 2 * STAGES;   // [ACC_BUFS] MMA -> epilogue
  uint64_t* tempty = bars + 2 * STAGES + 2;  // [ACC_BUFS] epilogue -> MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // a pair runs one tile sequence: unit = cluster index, rank = this CTA's half of each tile
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int unit = PAIR ? (int)cluster_id_x() : (int)blockIdx.x;
  const int n_units = PAIR ? (int)cluster_count_x() : (int)gridDim.x;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < ACC_BUFS; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), T::EPI_WARPS * (PAIR ? 2 : 1));  // both CTAs' epilogues drain the pair's accumulator
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.a);
    for (int i = 0; i < p.nb; ++i) prefetch_tmap(&maps.b[i]);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int kblocks = p.K / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer --
      int stage = 0;
      uint32_t phase = 0;
      for (int t = unit; t < p.num_tiles; t += n_units) {
        const int tile = GEN ? t % tiles : t, kb0 = GEN ? (t / tiles) * p.kb_slice : 0;
        const int kb1 = GEN && kb0 + p.kb_slice < kblocks ? kb0 + p.kb_slice : kblocks;
        const int m0 = (tile / p.n_tiles_n) * TM + (int)rank * 128;  // this CTA's first row
        const int n0 = (tile % p.n_tiles_n) * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&empty[stage]), phase ^ 1, p.err, abort_flag, wait_site(kSiteGemm, 1, 1))) goto producer_done;
          uint32_t fb = smem_u32(&full[stage]);
          if constexpr (PAIR) {
            // the even CTA's barrier counts both CTAs' bytes; the odd CTA only adds its copies
            if (rank == 0) mbar_arrive_expect_tx(fb, 2 * STAGE_BYTES);
            fb = mapa_shared(fb, 0);
          } else {
            mbar_arrive_expect_tx(fb, STAGE_BYTES);
          }
          uint8_t* sa = smem + stage * STAGE_BYTES;
          const int ka = a_kwrap ? (kb * BK) % a_kwrap : kb * BK;
          const int kbx = b_kwrap ? (kb * BK) % b_kwrap : kb * BK;
#pragma unroll
          for (int h = 0; h < MH; ++h) {
            if (a_mn) {  // two 64-row chunks of M, each [64 K][64 M]
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                const uint32_t dst = smem_u32(sa + h * A_HALF_BYTES + c * MN_CHUNK_BYTES);
                if constexpr (PAIR) tma_load_2d_pair(dst, &maps.a, fb, m0 + h * T::HS + c * 64, ka);
                else tma_load_2d(dst, &maps.a, fb, m0 + h * T::HS + c * 64, ka);
              }
            } else {
              if constexpr (PAIR) tma_load_2d_pair(smem_u32(sa + h * A_HALF_BYTES), &maps.a, fb, ka, m0 + h * T::HS);
              else tma_load_2d(smem_u32(sa + h * A_HALF_BYTES), &maps.a, fb, ka, m0 + h * T::HS);
            }
          }
#pragma unroll
          for (int h = 0; h < T::B_ROWS / 128; ++h) {
            const int row = n0 + (PAIR ? (int)rank : h) * 128;
            int mi = p.nb - 1, r = p.nrows[p.nb - 1];  // past the end: zero fill
            if (row < p.N) {
              mi = 0;
              while (mi + 1 < p.nb && row >= p.row_start[mi + 1]) ++mi;
              r = row - p.row_start[mi];
            }
            if (b_mn) {  // one B matrix stored [K][N]: two 64-column chunks of N, each [64 K][64 N]
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                const uint32_t dst = smem_u32(sa + A_BYTES + h * (128 * BK * 2) + c * MN_CHUNK_BYTES);
                if constexpr (PAIR) tma_load_2d_pair(dst, &maps.b[0], fb, row + c * 64, kbx);
                else tma_load_2d(dst, &maps.b[0], fb, row + c * 64, kbx);
              }
            } else {
              if constexpr (PAIR) tma_load_2d_pair(smem_u32(sa + A_BYTES + h * (128 * BK * 2)), &maps.b[mi], fb, kbx, r);
              else tma_load_2d(smem_u32(sa + A_BYTES + h * (128 * BK * 2)), &maps.b[mi], fb, kbx, r);
            }
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    producer_done:;
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // ------------------------------------------------------ MMA issuer --
      // Every lane runs this loop and its bounded waits; elect_one_sync picks the lane that issues
      // each tcgen05 instruction (issuing from a lane-divergent branch costs more per MMA).
      const uint32_t idesc = idesc_f32acc(PAIR ? 256 : 128, BN, a_mn, b_mn, p.in_fmt);
      // descriptors built once; a stage step adds STAGE_BYTES / 16 to the start address, a K = 16 step 2
      // (K-major: 32 bytes along the row) or 128 (MN-major: 16 rows of 128 bytes); MN-major operands
      // carry LBO = the 64-wide chunk's bytes (it lives in the low word), SBO = 8 rows either way
      const uint32_t d_hi = desc_hi(smem_desc_sw128(smem_u32(smem), 16, 1024));
      const uint32_t a_lo0 = desc_lo(smem_desc_sw128(smem_u32(smem), a_mn ? MN_CHUNK_BYTES : 16, 1024));
      const uint32_t b_lo0 = desc_lo(smem_desc_sw128(smem_u32(smem + A_BYTES), b_mn ? MN_CHUNK_BYTES : 16, 1024));
      const uint32_t a_kstep = a_mn ? 128 : 2, b_kstep = b_mn ? 128 : 2;
      int stage = 0;
      uint32_t phase = 0;
      int i = 0;
      for (int t = unit; t < p.num_tiles; t += n_units, ++i) {
        const int acc = i % ACC_BUFS;
        const uint32_t tph = (i / ACC_BUFS) & 1;
        if (!mbar_wait_bounded(smem_u32(&tempty[acc]), tph ^ 1, p.err, abort_flag, wait_site(kSiteGemm, 2, 2))) goto mma_done;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        const int kb0 = GEN ? (t / tiles) * p.kb_slice : 0;
        const int kb1 = GEN && kb0 + p.kb_slice < kblocks ? kb0 + p.kb_slice : kblocks;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&full[stage]), phase, p.err, abort_flag, wait_site(kSiteGemm, 2, 3))) goto mma_done;
          tc_fence_after();
          const uint32_t a_lo = a_lo0 + stage * (STAGE_BYTES >> 4);
          const uint32_t b_lo = b_lo0 + stage * (STAGE_BYTES >> 4);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
#pragma unroll
            for (int h = 0; h < MH; ++h) {  // rows h*128.. of the tile -> accumulator columns h*256..
              if constexpr (PAIR) {
                if (elect_one_sync()) umma_ss_pair_lohi(d_tmem + h * BN, a_lo + h * (A_HALF_BYTES >> 4) + a_kstep * k, d_hi,
                                                        b_lo + b_kstep * k, d_hi, idesc, (kb != kb0 || k != 0));
              } else {
                if (elect_one_sync()) umma_ss_lohi(d_tmem + h * BN, a_lo + h * (A_HALF_BYTES >> 4) + a_kstep * k, d_hi,
                                                   b_lo + b_kstep * k, d_hi, idesc, (kb != kb0 || k != 0));
              }
            }
          if constexpr (PAIR) {
            if (elect_one_sync()) umma_commit_pair(smem_u32(&empty[stage]), 3);
          } else {
            if (elect_one_sync()) umma_commit(smem_u32(&empty[stage]));
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if constexpr (PAIR) {
          if (elect_one_sync()) umma_commit_pair(smem_u32(&tfull[acc]), 3);
        } else {
          if (elect_one_sync()) umma_commit(smem_u32(&tfull[acc]));
        }
      }
    mma_done:;
    }
  } else {
    // --------------------------------------------------------- epilogue --
    const int quad = warp & 3;        // this warp may touch TMEM lanes [32*quad, 32*quad+32)
    const int half = (warp - 2) / 4;  // MH = 2: which 128-row half of the tile (accumulator columns half*256..)
    uint8_t* stg = staging + (warp - 2) * T::EPI_BUFS * T::STG_BYTES;
    int sbuf = 0;
    bool bad = false;
    // side job while the first accumulator fills: this CTA's share of the fp16 copies, 8 elements
    // per 16-byte vector (the sizes are multiples of 8)
    for (int i = 0; i < 2; ++i) {
      const long long nvec = p.side_n[i] / 8;
      const long long chunk = (nvec + gridDim.x - 1) / gridDim.x;
      const long long lo = blockIdx.x * chunk, hi = lo + chunk < nvec ? lo + chunk : nvec;
      for (long long e = lo + (threadIdx.x - 64); e < hi; e += 32 * T::EPI_WARPS) {
        const uint4 raw = *reinterpret_cast<const uint4*>(p.side_src[i] + e * 8);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
        uint32_t h[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(b2[k]);
          const float fx = f.x * p.side_scale, fy = f.y * p.side_scale;
          bad |= f16_overflow(fx) || f16_overflow(fy);
          h[k] = pack_f16x2(fx, fy);
        }
        *reinterpret_cast<uint4*>(p.side_dst[i] + e * 8) = make_uint4(h[0], h[1], h[2], h[3]);
      }
    }
    int i = 0;
    for (int t = unit; t < p.num_tiles; t += n_units, ++i) {
      const int acc = i % ACC_BUFS;
      const uint32_t tph = (i / ACC_BUFS) & 1;
      if (!mbar_wait_bounded(smem_u32(&tfull[acc]), tph, p.err, abort_flag, wait_site(kSiteGemm, 3, 4))) break;
      tc_fence_after();
      const int tile = GEN ? t % tiles : t;
      const long long m0 = (long long)(tile / p.n_tiles_n) * TM + rank * 128;
      const int n0 = (tile % p.n_tiles_n) * BN;
      const long long row0 = m0 + half * T::HS + quad * 32;  // this warp's 32 rows
      const long long row = row0 + lane;
      const uint32_t col0 = tmem_base + ((uint32_t)(quad * 32) << 16) + (acc + half) * BN;
      if (T::EPI_BUFS > 0 && p.tma_store) {
        const bool h = p.out_type == (int)DType::F16;
#pragma unroll 1
        for (int c = 0; c < BN / 64; ++c) {
          uint32_t r[64];
          tmem_ld_32x32b_x32(col0 + c * 64, r);
          tmem_ld_32x32b_x32(col0 + c * 64 + 32, r + 32);
          tmem_ld_wait();
          if (p.v_cache != nullptr && n0 + c * 64 >= p.v_col0) {  // v~: the value shift, stored directly
            if (row < p.M && n0 + c * 64 < p.N) bad |= store_value_shift(p, row, n0 + c * 64 - p.v_col0, r);
            continue;
          }
          uint32_t w[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float x0 = u2f(r[2 * e]), x1 = u2f(r[2 * e + 1]);
            if (h) {
              w[e] = pack_f16x2(x0, x1);
              bad |= f16_overflow(x0) || f16_overflow(x1);
            } else {
              w[e] = pack_bf16x2(x0, x1);
            }
          }
          // the buffer's previous store has read it; row `lane`, 16-byte chunk j at j ^ (lane % 8)
          if (lane == 0) bulk_wait_read<T::EPI_BUF_COUNT - 1>();
          __syncwarp();
          uint8_t* buf = stg + sbuf * T::STG_BYTES;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          fence_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < p.M) {  // rows past M and columns past N are clipped by the map
            tma_store_2d(&maps.c, smem_u32(buf), n0 + c * 64, (int)row0);
            bulk_commit();
          }
          sbuf = sbuf + 1 == T::EPI_BUF_COUNT ? 0 : sbuf + 1;
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(col0 + c * 32, r);
          tmem_ld_wait();
          const int col = n0 + c * 32;
          if (p.v_cache != nullptr && col >= p.v_col0) {  // v~: the value shift, 64 columns at a time
            uint32_t r2[32];
            tmem_ld_32x32b_x32(col0 + c * 32 + 32, r2);
            tmem_ld_wait();
            uint32_t rr[64];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              rr[e] = r[e];
              rr[32 + e] = r2[e];
            }
            if (row < p.M && col < p.N) bad |= store_value_shift(p, row, col - p.v_col0, rr);
            ++c;
            continue;
          }
          if (row < p.M && col < p.N) bad |= store_row_chunk(p, row, col, r);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
        else mbar_arrive(smem_u32(&tempty[acc]));
      }
    }
    if (lane == 0) bulk_wait_all();  // the staging buffers stay valid until the stores are done
    report_range(bad, p.err);
  }
  tc_fence_before();
  __syncthreads();
  // after a wait of this CTA timed out, copies and MMAs it issued may still be landing in its shared
  // and tensor memory: give them a bounded 20 us before that memory is released
  if (*abort_flag) {
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 20000ull) {
    }
  }
  // a pair leaves together: no remote arrival or MMA of one CTA is still pending on the other
  if constexpr (PAIR) cluster_sync_all();
  tc_fence_after();
  if (warp == 1) {
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// 2D map of a row-major 16-bit matrix, 128-byte swizzle; row_bytes = 0 for densely packed rows.
bool encode_2d(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
               uint32_t box_inner, uint32_t box_outer, uint64_t row_bytes = 0) {
  EncodeTiledFn enc = get_encode_tiled();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes ? row_bytes : inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int gemm_tc_ksplit(long long M, int N, int K) {
  const long long tiles = ((M + 255) / 256) * ((N + 255) / 256);
  const long long units = num_sms() / 2;
  if (tiles >= units) return 1;  // a full round of tiles already: slices would only add reductions
  // The makespan of ks slices in K blocks per CTA pair: rounds of work items times blocks per slice
  // (the launch evens the slices out the same way). Of the counts within 3 % of the shortest, the
  // fewest slices (fewer fp32 reductions).
  const long long kblocks = K / 64, kmax = K / 256;
  auto cost = [&](long long ks) {
    const long long slice = (kblocks + ks - 1) / ks, n = (kblocks + slice - 1) / slice;
    return ((tiles * n + units - 1) / units) * slice;
  };
  long long best = cost(1);
  for (long long ks = 2; ks <= kmax; ++ks) best = cost(ks) < best ? cost(ks) : best;
  for (long long ks = 1; ks <= kmax; ++ks)
    if (100 * cost(ks) <= 103 * best) return (int)ks;
  return 1;
}

namespace {
template <int MH, bool GEN>
cudaError_t launch_single(int grid, const GemmMaps& maps, const GemmParams& p, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<MH, false, GEN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Shape<MH>::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  gemm_tc_kernel<MH, false, GEN><<<grid, Shape<MH>::NUM_THREADS, Shape<MH>::SMEM_BYTES, stream>>>(maps, p);
  return cudaGetLastError();
}
}  // namespace

bool gemm_tc_supported(long long M, int N, int K) {
  return M >= 1 && M < (1ll << 31) && K >= BK && K % BK == 0 && N >= 128 && N % 128 == 0;
}

namespace {
template <int MH>
void pair_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr, int grid, cudaStream_t stream) {
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(Shape<MH, true>::NUM_THREADS);
  cfg.dynamicSmemBytes = Shape<MH, true>::SMEM_BYTES;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
}
// How many two-CTA clusters of the pair kernel fit on the device at once (0: the pair form is not
// used). Queried once per process on the current device.
template <int MH>
int pair_clusters() {
  static const int n = [] {
    if (cudaFuncSetAttribute(gemm_tc_kernel<MH, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Shape<MH, true>::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(gemm_tc_kernel<MH, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Shape<MH, true>::SMEM_BYTES) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    pair_config<MH>(cfg, attr, 2 * (num_sms() / 2), nullptr);
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, gemm_tc_kernel<MH, true, false>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    return c;
  }();
  return n;
}
}  // namespace

cudaError_t launch_gemm_tc(const GemmTcArgs& a, cudaStream_t stream) {
  int N = 0;
  for (int i = 0; i < a.nb; ++i) {
    if (a.nrows[i] % 128 != 0) return cudaErrorInvalidValue;
    N += a.nrows[i];
  }
  if (!gemm_tc_supported(a.M, N, a.K) || a.nb < 1 || a.nb > 3) return cudaErrorInvalidValue;
  if (a.ldc % 8 != 0 || (reinterpret_cast<uintptr_t>(a.C) & 15) != 0) return cudaErrorInvalidValue;
  if (a.in != DType::BF16 && a.in != DType::F16) return cudaErrorInvalidValue;
  const CUtensorMapDataType dt =
      a.in == DType::F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  GemmMaps maps;
  GemmParams p{};
  // an operand that repeats along K (its own extent whole 64-deep blocks, at most K)
  for (const int w : {a.a_kwrap, a.b_kwrap})
    if (w < 0 || (w > 0 && (w % BK != 0 || w > a.K))) return cudaErrorInvalidValue;
  p.a_kwrap = a.a_kwrap;
  p.b_kwrap = a.b_kwrap;
  p.a_mn = a.a_mn ? 1 : 0;
  p.b_mn = a.b_mn ? 1 : 0;
  if (p.b_mn && a.nb != 1) return cudaErrorInvalidValue;
  if ((a.lda != 0 && (a.lda * 2) % 16 != 0) || (a.ldb != 0 && (a.ldb * 2) % 16 != 0)) return cudaErrorInvalidValue;
  // the maps' K extents: what the operand holds (kext), else its wrap period, else K; columns of a
  // period past the operand's extent read zeros
  const int ka = a.a_kext ? a.a_kext : (a.a_kwrap ? a.a_kwrap : a.K);
  const int kb_ext = a.b_kext ? a.b_kext : (a.b_kwrap ? a.b_kwrap : a.K);
  if (a.a_kext < 0 || a.b_kext < 0 || (a.a_kext > 0 && a.a_kext > (a.a_kwrap ? a.a_kwrap : a.K)) ||
      (a.b_kext > 0 && a.b_kext > (a.b_kwrap ? a.b_kwrap : a.K)))
    return cudaErrorInvalidValue;
  // K-major: [M][K] rows of K; MN-major: [K][M] rows of M, 64 x 64 boxes (row strides lda / ldb)
  if (p.a_mn ? !encode_2d(&maps.a, a.A, dt, (uint64_t)a.M, (uint64_t)ka, 64, BK, (uint64_t)a.lda * 2)
             : !encode_2d(&maps.a, a.A, dt, (uint64_t)ka, (uint64_t)a.M, BK, 128, (uint64_t)a.lda * 2))
    return cudaErrorInvalidValue;
  int start = 0;
  for (int i = 0; i < 3; ++i) {
    const int src = i < a.nb ? i : 0;
    if (p.b_mn ? !encode_2d(&maps.b[i], a.B[src], dt, (uint64_t)a.nrows[src], (uint64_t)kb_ext, 64, BK,
                            (uint64_t)a.ldb * 2)
               : !encode_2d(&maps.b[i], a.B[src], dt, (uint64_t)kb_ext, (uint64_t)a.nrows[src], BK, 128))
      return cudaErrorInvalidValue;
    p.row_start[i] = i < a.nb ? start : N;
    p.nrows[i] = a.nrows[src];
    if (i < a.nb) start += a.nrows[i];
  }
  p.M = a.M;
  p.N = N;
  p.K = a.K;
  p.nb = a.nb;
  p.C = a.C;
  p.ldc = a.ldc;
  p.out_type = (int)a.out;
  p.in_fmt = a.in == DType::F16 ? kFmtF16 : kFmtBF16;
  for (int i = 0; i < 2; ++i) {
    if (a.side_n[i] > 0 && (a.side_n[i] % 8 != 0 || (reinterpret_cast<uintptr_t>(a.side_src[i]) & 15) != 0 ||
                            (reinterpret_cast<uintptr_t>(a.side_dst[i]) & 15) != 0))
      return cudaErrorInvalidValue;
    p.side_src[i] = static_cast<const __nv_bfloat16*>(a.side_src[i]);
    p.side_dst[i] = static_cast<__half*>(a.side_dst[i]);
    p.side_n[i] = a.side_n[i] > 0 ? a.side_n[i] : 0;
  }
  p.side_scale = a.side_scale != 0.f ? a.side_scale : 1.f;
  if (a.v_cache != nullptr) {
    // 64-column groups of v~ start on a 64-column boundary and never straddle the shifted half
    if (a.v_col0 % 64 != 0 || a.Lkv % 128 != 0 || a.vfrom % 64 != 0 || a.S < 1 || a.v_col0 + a.Lkv != N ||
        a.out != DType::F16 ||
        ((reinterpret_cast<uintptr_t>(a.v_cache) | reinterpret_cast<uintptr_t>(a.v_att)) & 15) != 0)
      return cudaErrorInvalidValue;
    p.v_cache = static_cast<__nv_bfloat16*>(a.v_cache);
    p.v_att = static_cast<__half*>(a.v_att);
    p.v_col0 = a.v_col0;
    p.Lkv = a.Lkv;
    p.S = a.S;
    p.vshift = a.vshift;
    p.vfrom = a.vfrom;
  }
  // 256-row tiles keep direct stores: their single accumulator leaves nothing to overlap the wait
  // for a staging buffer with, while direct stores retire without waiting
  // Pairs whenever a 256-row tile has rows to fill (on this workload's projections: 37.0 -> 34.9 us
  // and 63.7 -> 61.6 us against the single-CTA forms; 256 rows per CTA of a pair measured the same)
  const bool pair = a.M >= 256 && pair_clusters<1>() > 0;
  const bool big = !pair && a.K >= 1024 && a.M >= 256;
  p.tma_store = !big && (a.out == DType::BF16 || a.out == DType::F16);
  if (p.tma_store) {
    const CUtensorMapDataType ct =
        a.out == DType::F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!encode_2d(&maps.c, a.C, ct, (uint64_t)N, (uint64_t)a.M, 64, 32, (uint64_t)a.ldc * 2))
      return cudaErrorInvalidValue;
  }
  p.err = a.dev_err;
  p.n_tiles_n = (N + BN - 1) / BN;
  // 256-row tiles (one CTA, or a pair) when the main loop is long enough to carry the epilogue
  const int TM = big || pair ? 256 : 128;
  const long long m_tiles = (a.M + TM - 1) / TM;
  p.tiles = (int)(m_tiles * p.n_tiles_n);
  const int kblocks = a.K / BK;
  int ks = a.ksplit > 1 ? a.ksplit : 1;
  if (ks > kblocks) ks = kblocks;
  if (ks > 1 && (a.out != DType::F32 || a.v_cache != nullptr || a.side_n[0] > 0 || a.side_n[1] > 0))
    return cudaErrorInvalidValue;
  p.kb_slice = (kblocks + ks - 1) / ks;
  p.ksplit = (kblocks + p.kb_slice - 1) / p.kb_slice;  // no empty slice
  p.num_tiles = p.tiles * p.ksplit;
  const bool gen = p.ksplit > 1 || p.a_kwrap || p.b_kwrap || p.a_mn || p.b_mn;
  if (pair) {
    const int clusters = p.num_tiles < pair_clusters<1>() ? p.num_tiles : pair_clusters<1>();
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    pair_config<1>(cfg, attr, 2 * clusters, stream);
    return gen ? cudaLaunchKernelEx(&cfg, gemm_tc_kernel<1, true, true>, maps, p)
               : cudaLaunchKernelEx(&cfg, gemm_tc_kernel<1, true, false>, maps, p);
  }
  const int grid = p.num_tiles < num_sms() ? p.num_tiles : num_sms();
  if (big) return gen ? launch_single<2, true>(grid, maps, p, stream) : launch_single<2, false>(grid, maps, p, stream);
  return gen ? launch_single<1, true>(grid, maps, p, stream) : launch_single<1, false>(grid, maps, p, stream);
}

}  // namespace cca
