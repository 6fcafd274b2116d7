// Latent preprocessing of one CCA / CCGQA block (steps a2-a8: seq conv, channel conv, QK-mean
// before and after, RoPE, value shift, KV-cache write) for bf16 blocks with head_dim 128 whose
// QK-mean includes the after-conv term: a persistent, warp-specialised tcgen05 kernel.
//
// "Compressed Convolutional Attention" (gist.science/es/paper/2510.04476), section 2.B items 1-3
// and section 3 item 2; the forms follow the readings the other preprocessing kernels take
// (depthwise causal seq conv with tap K-1 on the current token, per-head dense channel mix, both
// QK-mean terms added to the conv outputs, rotate-half RoPE, upper half of the V latent shifted
// by one token).
//
// Work unit: a tile of 128 tokens of one sequence x one KV group (its K head and its G query
// heads). One CTA per SM walks its tiles; inside it each role has its own warps, so that loading,
// the seq conv, the tensor-core MMAs, the per-row epilogue and the stores of consecutive heads
// overlap:
//   warp 0      loader:   per tile the RoPE base angles and the group's seq taps; per head the
//                         fp16 latents (128 rows + a K-1 row halo, TMA into a 2-slot ring) and
//                         the head's channel-mix weights (TMA)
//   warp 1      MMA:      one elected lane issues the head's tcgen05 MMAs into tensor memory
//   warp 2      storer:   TMA tensor stores of q, the fp16 attention copy of k and the bf16 cache
//   warps 3-6   conv:     thread = one 8-channel chunk of 16 consecutive token rows, the latent
//                         rows sliding through registers; the causal seq conv in fp32, rounded to
//                         fp16 into the K-major 128-byte-swizzled A operand; then the value shift
//   warps 7-14  epilogue: two threads per token row (= TMEM lane), 32 RoPE pairs each, whose
//                         (cos, sin) stay in registers for all heads of the tile; combine, RoPE;
//                         q is staged in the head's s slot once its MMAs have read it
//
// With P = the after-conv QK-mean bit (set for this kernel) and R = the before-conv bit, the
// block's q and k are linear in the conv outputs c_q = s_q W^T, c_k and the raw latents q~, k~:
//   q_h = 1.5 c_q,h + R/2 q~_h + 1/2 c_k + R/2 k~
//   k   = 1.5 c_k + R/2 k~ + R/(2G) sum_h q~_h + 1/(2G) sum_h c_q,h
// so the tensor cores accumulate all of it, with the channel weights scaled by 1.5 (the fp16
// copies are made scaled; exact for bf16 weights in fp16's normal range) and the latent terms as
// MMAs of the raw latent tile by small scaled identity tiles (N = 16, exact):
//   ACK   = s_K (1.5 W_K)^T + k~ (1.5 R I)                          = 1.5 c_k + 1.5 R k~
//   S     = k~ (-3 G R I) + sum_h [ s_h (1.5 W_h)^T + q~_h (1.5 R I) ]
//   ACQ_h = s_h (1.5 W_h)^T + q~_h (R/2 I)                          = 1.5 c_q,h + R/2 q~_h
// and the epilogue reads only tensor memory: q_h = ACQ_h + ACK / 3, k = ACK + S / (3 G).
// Tensor memory (512 columns): ACK | S | ACQ (two buffers). The K head's epilogue releases ACK and
// S as soon as it has read them (so the next tile's MMAs need not wait for its stores); its outputs
// are staged in a buffer of their own, the fp16 attention copy first, while the bf16 cache values
// wait in the last query head's ACQ columns. Shared memory holds two latent slots and two s slots;
// the channel weights have one slot of two K-halves, each released as soon as the MMAs that read it
// are done, so that the next head's first half lands while the current head's second half is used.
//
// Every mbarrier wait is bounded; on expiry the CTA records the wait site, every role leaves its
// loop, copies and MMAs in flight get a bounded 20 us to land, and the tensor memory is freed.
#include <math.h>

#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

constexpr int D = 128;
constexpr int TT = 128;           // tokens per tile (one TMEM lane each)
constexpr int KMAX = 8;           // seq-conv taps: a halo of up to 7 rows
constexpr int GMAX = 8;
constexpr int NWARP = 15;
constexpr int NEPI = 256;              // epilogue threads
constexpr int NT = NWARP * 32;
constexpr int W_LOAD = 0, W_MMA = 1, W_STORE = 2, W_CONV0 = 3, W_EPI0 = 7;
constexpr int HALF = 16384;            // one 64-column half of a 128 x 128 16-bit tile
constexpr int TILE = 2 * HALF;
constexpr int HALO_HALF = 1024;        // up to 8 halo rows of one 64-column half
constexpr int LAT_SLOT = TILE + 2 * HALO_HALF;
constexpr int IDT = 2048;              // 16 rows x 128 bytes: one identity B operand

// shared memory, from a 1024-byte-aligned base
constexpr int OFF_LAT = 0;                        // [2] latent slots: main tile, then two halo halves
constexpr int OFF_W = OFF_LAT + 2 * LAT_SLOT;     // channel weights of a head (two K-halves)
constexpr int OFF_SB = OFF_W + TILE;              // [2] s operands; a query head's q is staged in its own
constexpr int OFF_O = OFF_SB + 2 * TILE;          // the K head's outputs (fp16, then bf16)
constexpr int OFF_IDT = OFF_O + TILE;             // identity tiles: 0.5 I, 1.5 I, -3G I
constexpr int OFF_TAPS = OFF_IDT + 3 * IDT;       // [2] the seq taps of a tile's heads
static_assert(OFF_W % 1024 == 0 && OFF_SB % 1024 == 0 && OFF_O % 1024 == 0 && OFF_IDT % 1024 == 0 &&
                  LAT_SLOT % 1024 == 0,
              "swizzled tiles start on 1024-byte boundaries");

constexpr uint32_t T_ACK = 0, T_S = 128, T_ACQ = 256;  // tensor-memory columns (ACQ: two buffers of 128)

// barriers
enum Bar : int {
  B_LAT_FULL = 0,   // [2]
  B_LAT_FREE = 2,   // [2]
  B_W_FULL = 4,     // [2] per K-half of the weight slot
  B_W_FREE = 6,     // [2] per K-half
  B_TAPS_FULL = 8,  // [2]
  B_TAPS_FREE = 10, // [2]
  B_RTAB_FULL = 12, // [2]
  B_RTAB_FREE = 14, // [2]
  B_S_FULL = 16,    // [2]
  B_S_FREE = 18,    // [2]
  B_ACK_FULL = 20,
  B_ACK_FREE = 21,
  B_ACQ_FULL = 22,  // [2]
  B_ACQ_FREE = 24,  // [2]
  B_STAGED = 26,    // [2] a query head's q is staged in its s slot
  B_O_STAGED = 28,  // the K head's fp16 copy, then its bf16 cache values, are staged
  B_O_FREE = 29,    // the fp16 copy has left the staging buffer
  NBAR = 30
};

__host__ __device__ constexpr int taps_bytes(int H1, int K) { return ((H1 * D * K * 2) + 15) & ~15; }
__host__ __device__ constexpr int off_rtab(int H1, int K) { return OFF_TAPS + 2 * taps_bytes(H1, K); }
__host__ __device__ constexpr int off_thf(int H1, int K) { return off_rtab(H1, K) + 2 * 64 * 8; }
__host__ __device__ constexpr int off_bar(int H1, int K) { return off_thf(H1, K) + 64 * 4; }
__host__ __device__ constexpr int smem_bytes(int H1, int K) { return off_bar(H1, K) + NBAR * 8 + 16 + 1024; }
constexpr int kSmemLimit = 232448;

struct Theta {
  double v[D / 2];  // base^(-2i/d)
};

struct WsMaps {
  CUtensorMap lat;   // [B][S][Nlat] fp16, box 64 x 128 x 1 (main rows)
  CUtensorMap halo;  // [B][S][Nlat] fp16, box 64 x (K-1) x 1
  CUtensorMap wc;    // [(nq+nkv)*D][D] fp16 channel weights (scaled by 1.5), box 64 x 128
  CUtensorMap q;     // [B][S][Lq] fp16 (store)
  CUtensorMap ka;    // [B][S][Lkv] fp16 attention copy of k (store)
  CUtensorMap kc;    // [B][S][Lkv] bf16 K cache (store)
};

struct WsParams {
  const __half* lat;  // [T, Nlat] (value shift reads)
  __half* q;          // [T, Lq]
  const __nv_bfloat16 *cq_seq, *ck_seq;
  __nv_bfloat16* v_cache;   // [T, Lkv]
  __half* v_att;            // [T, Lkv]
  const __nv_bfloat16* wo;  // [E, Lq]: fp16 copy made here as a side job
  __half* wo_lat;
  long long wo_n;
  unsigned* err;
  int* zero_cnt;  // split-pair counters of the attention launch that follows (cleared here)
  int B, S, nq, nkv, K, pre, vshift, vfrom, use_rope;
  int v_done;  // the down-projection's epilogue has written the V cache and its attention copy
  int ntiles, nT;
};

// global -> shared bulk copy (no tensor map), completing on an mbarrier
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_x8(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// Byte offset of the 16-byte chunk `c` (8 columns, 0..15) of `row` in a 128-column 16-bit tile
// stored as two 64-column halves of 128-byte rows with the 128-byte swizzle (the layout of a TMA
// box with SWIZZLE_128B and of a K-major tcgen05 operand).
__device__ __forceinline__ uint32_t chunk_off(int row, int c) {
  return (uint32_t)((c >> 3) * HALF + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

__device__ __forceinline__ void spin_ns(unsigned long long ns) {
  const unsigned long long t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 < ns) {
  }
}

struct TileId {
  int b, t0, g;
};
__device__ __forceinline__ TileId tile_of(const WsParams& p, int u) {
  TileId t;
  t.g = u % p.nkv;
  const int rest = u / p.nkv;
  t.t0 = (rest % p.nT) * TT;
  t.b = rest / p.nT;
  return t;
}

// Causal seq conv of one head, one thread: the 8 channels of chunk c (0..15) for the 16 token rows
// rb*16 .. rb*16+15 of the tile. Output row t is sum_j w[ch][j] z[t - (K-1) + j][ch]; the latent rows
// slide through registers, so each staged row is read once; rows before the tile come from the halo.
template <int KC>
__device__ __forceinline__ void seq_conv_chunk(const uint8_t* lat, const uint8_t* halo, uint8_t* sdst,
                                               const __nv_bfloat16* taps, int K, int c, int rb) {
  constexpr int KM = KC > 0 ? KC : KMAX;
  const int KK = KC > 0 ? KC : K;
  // the chunk's taps: 8 channels x K, contiguous (16 K bytes)
  float w[8][KM];
  {
    const uint4* tv = reinterpret_cast<const uint4*>(taps + (size_t)c * 8 * KK);
#pragma unroll
    for (int q = 0; q < KM; ++q) {
      if (KC == 0 && q >= KK) break;
      const uint4 v = tv[q];
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(b2[e]);
        // element 8q + 2e + {0,1} of the chunk's [8][K] taps
        const int a = 8 * q + 2 * e;
        w[a / KK][a % KK] = f.x;
        w[(a + 1) / KK][(a + 1) % KK] = f.y;
      }
    }
  }
  auto load_row = [&](int src, float* z) {
    const uint8_t* ptr = src >= 0 ? lat + chunk_off(src, c)
                                  : halo + (c >> 3) * HALO_HALF + (src + KK - 1) * 128 +
                                        (((c & 7) ^ ((src + KK - 1) & 7)) << 4);
    const uint4 v = *reinterpret_cast<const uint4*>(ptr);
    const __half2* h2 = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __half22float2(h2[q]);
      z[2 * q] = f.x;
      z[2 * q + 1] = f.y;
    }
  };
  const int r0 = rb * 16;
  float win[KM][8];  // win[j]: row t - (K-1) + j of the current output row t
#pragma unroll
  for (int j = 0; j + 1 < KM; ++j)
    if (j + 1 < KK) load_row(r0 - (KK - 1) + j, win[j]);
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    load_row(r0 + t, win[KK - 1]);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (j < KK) fma2(a0, a1, w[e][j], w[e + 1][j], win[j][e], win[j][e + 1], a0, a1);
      acc[e] = a0;
      acc[e + 1] = a1;
    }
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) o[q] = pack_f16x2(acc[2 * q], acc[2 * q + 1]);
    *reinterpret_cast<uint4*>(sdst + chunk_off(r0 + t, c)) = make_uint4(o[0], o[1], o[2], o[3]);
#pragma unroll
    for (int j = 0; j + 1 < KM; ++j)
      if (j + 1 < KK)
#pragma unroll
        for (int e = 0; e < 8; ++e) win[j][e] = win[j + 1][e];
  }
}

template <int KC>
__global__ void __launch_bounds__(NT, 1) preproc_ws_kernel(const __grid_constant__ WsMaps maps,
                                                          const __grid_constant__ WsParams p,
                                                          const __grid_constant__ Theta th) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int G = p.nq / p.nkv, H1 = G + 1, K = KC > 0 ? KC : p.K;
  const int Lq = p.nq * D, Lkv = p.nkv * D, Nlat = Lq + 2 * Lkv;
  const int TAPS = taps_bytes(H1, K);
  float2* rtab = reinterpret_cast<float2*>(smem + off_rtab(H1, K));  // [2][64] (cos, sin) of t0 theta_i
  float* thf = reinterpret_cast<float*>(smem + off_thf(H1, K));      // theta_i in fp32
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + off_bar(H1, K));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool pre = p.pre != 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_LAT_FULL + i), 1);
      mbar_init(bar(B_LAT_FREE + i), 1);
      mbar_init(bar(B_TAPS_FULL + i), 1);
      mbar_init(bar(B_TAPS_FREE + i), 128);
      mbar_init(bar(B_RTAB_FULL + i), 32);
      mbar_init(bar(B_RTAB_FREE + i), NEPI);
      mbar_init(bar(B_S_FULL + i), 128);
      mbar_init(bar(B_S_FREE + i), 2);  // the MMAs have read s, and the storer the q staged there
      mbar_init(bar(B_STAGED + i), NEPI);
      mbar_init(bar(B_ACQ_FULL + i), 1);
      mbar_init(bar(B_ACQ_FREE + i), NEPI);
      mbar_init(bar(B_W_FULL + i), 1);
      mbar_init(bar(B_W_FREE + i), 1);
    }
    mbar_init(bar(B_ACK_FULL), 1);
    mbar_init(bar(B_ACK_FREE), NEPI);
    mbar_init(bar(B_O_STAGED), NEPI);
    mbar_init(bar(B_O_FREE), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // identity B operands (16 rows of the 128-byte-swizzled K-major layout; entry (n, n) of the
  // first 16 columns): 0.5 I, 1.5 I, -3G I
  if (threadIdx.x >= 64) {
    for (int e = threadIdx.x - 64; e < 3 * IDT / 16; e += NT - 64)
      *reinterpret_cast<uint4*>(smem + OFF_IDT + e * 16) = make_uint4(0, 0, 0, 0);
  }
  if (threadIdx.x < 64 && threadIdx.x < D / 2) thf[threadIdx.x] = (float)th.v[threadIdx.x];
  if (warp == W_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  __syncthreads();
  if (threadIdx.x < 48) {
    const int k = threadIdx.x / 16, n = threadIdx.x % 16;
    const float v = k == 0 ? 0.5f : (k == 1 ? 1.5f : -3.0f * (float)G);
    const uint32_t off = OFF_IDT + k * IDT + n * 128 + ((((n >> 3) ^ (n & 7))) << 4) + (n & 7) * 2;
    *reinterpret_cast<__half*>(smem + off) = __float2half_rn(v);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == W_LOAD) {
    // ------------------------------------------------------------------ loader --
    if (lane == 0) {
      prefetch_tmap(&maps.lat);
      if (K > 1) prefetch_tmap(&maps.halo);
      prefetch_tmap(&maps.wc);
    }
    const uint32_t lat_bytes = (uint32_t)(TILE + (K > 1 ? 2 * (K - 1) * 128 : 0));
    int kt = 0;
    for (int u = blockIdx.x; u < p.ntiles; u += gridDim.x, ++kt) {
      const TileId tl = tile_of(p, u);
      const int tb = kt & 1;
      if (kt >= 2 && !mbar_wait_bounded(bar(B_TAPS_FREE + tb), ((kt >> 1) & 1) ^ 1, p.err, abort_flag,
                                        wait_site(kSitePreWs, 0, 2)))
        break;
      if (lane == 0) {
        const uint32_t dst = sbase + OFF_TAPS + tb * TAPS;
        const uint32_t kb = (uint32_t)(D * K * 2), qb = (uint32_t)(G * D * K * 2);
        mbar_arrive_expect_tx(bar(B_TAPS_FULL + tb), kb + qb);
        bulk_load(dst, p.ck_seq + (size_t)tl.g * D * K, kb, bar(B_TAPS_FULL + tb));
        bulk_load(dst + kb, p.cq_seq + (size_t)tl.g * G * D * K, qb, bar(B_TAPS_FULL + tb));
      }
      bool ok = true;
      for (int i = 0; i < H1 && ok; ++i) {
        const int n = kt * H1 + i, x = n & 1;
        if (n >= 2 && !mbar_wait_bounded(bar(B_LAT_FREE + x), ((n >> 1) & 1) ^ 1, p.err, abort_flag,
                                         wait_site(kSitePreWs, 0, 3))) {
          ok = false;
          break;
        }
        const int col = i == 0 ? Lq + tl.g * D : (tl.g * G + i - 1) * D;
        if (lane == 0) {
          const uint32_t dst = sbase + OFF_LAT + x * LAT_SLOT;
          mbar_arrive_expect_tx(bar(B_LAT_FULL + x), lat_bytes);
          for (int h = 0; h < 2; ++h) tma_load_3d(dst + h * HALF, &maps.lat, bar(B_LAT_FULL + x), col + 64 * h, tl.t0, tl.b);
          if (K > 1)
            for (int h = 0; h < 2; ++h)
              tma_load_3d(dst + TILE + h * HALO_HALF, &maps.halo, bar(B_LAT_FULL + x), col + 64 * h, tl.t0 - (K - 1),
                          tl.b);
        }
        const int wrow = i == 0 ? (p.nq + tl.g) * D : (tl.g * G + i - 1) * D;
        for (int h = 0; h < 2 && ok; ++h) {
          if (n >= 1 && !mbar_wait_bounded(bar(B_W_FREE + h), (n - 1) & 1, p.err, abort_flag,
                                           wait_site(kSitePreWs, 0, 4))) {
            ok = false;
            break;
          }
          if (lane == 0) {
            mbar_arrive_expect_tx(bar(B_W_FULL + h), HALF);
            tma_load_2d(sbase + OFF_W + h * HALF, &maps.wc, bar(B_W_FULL + h), 64 * h, wrow);
          }
        }
        if (!ok) break;
        __syncwarp();
        if (i == 0) {
          // the tile's RoPE base angles, once its first copies are on their way
          if (kt >= 2 && !mbar_wait_bounded(bar(B_RTAB_FREE + tb), ((kt >> 1) & 1) ^ 1, p.err, abort_flag,
                                            wait_site(kSitePreWs, 0, 1))) {
            ok = false;
            break;
          }
          if (p.use_rope) {
            // (cos, sin) of t0 theta_i, the angle reduced modulo 2 pi in fp64
            for (int ii = lane; ii < D / 2; ii += 32) {
              const double a = (double)tl.t0 * th.v[ii];
              const double k = rint(a * 0.15915494309189535);
              double rr = fma(-k, 6.283185307179586, a);
              rr = fma(-k, 2.4492935982947064e-16, rr);
              float c, sn;
              sincosf((float)rr, &sn, &c);
              rtab[tb * 64 + ii] = make_float2(c, sn);
            }
          }
          mbar_arrive(bar(B_RTAB_FULL + tb));
        }
      }
      if (!ok) break;
    }
  } else if (warp == W_MMA) {
    // --------------------------------------------------------------------- MMA --
    const uint32_t id128 = idesc_f32acc(128, 128, 0, 0, kFmtF16);
    const uint32_t id16 = idesc_f32acc(128, 16, 0, 0, kFmtF16);
    const uint64_t wdesc = smem_desc_sw128(sbase + OFF_W, 16, 1024);
    const uint32_t hi = desc_hi(wdesc);
    const uint32_t idt_lo[3] = {desc_lo(smem_desc_sw128(sbase + OFF_IDT, 16, 1024)),
                                desc_lo(smem_desc_sw128(sbase + OFF_IDT + IDT, 16, 1024)),
                                desc_lo(smem_desc_sw128(sbase + OFF_IDT + 2 * IDT, 16, 1024))};
    // K step kk of a 128-column operand: 64-column half kk / 4 (16 KB apart), 32 bytes per step
    auto koff = [](int kk) { return (uint32_t)((kk >> 2) * (HALF >> 4) + (kk & 3) * 2); };
    int kt = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.ntiles && ok; u += gridDim.x, ++kt) {
      bool s_init = false;
      for (int i = 0; i < H1; ++i) {
        const int n = kt * H1 + i, x = n & 1;
        if (!mbar_wait_bounded(bar(B_S_FULL + x), (n >> 1) & 1, p.err, abort_flag, wait_site(kSitePreWs, 1, 5)) ||
            !mbar_wait_bounded(bar(B_LAT_FULL + x), (n >> 1) & 1, p.err, abort_flag, wait_site(kSitePreWs, 1, 6))) {
          ok = false;
          break;
        }
        const uint32_t s_lo = desc_lo(smem_desc_sw128(sbase + OFF_SB + x * TILE, 16, 1024));
        const uint32_t w_lo = desc_lo(smem_desc_sw128(sbase + OFF_W, 16, 1024));
        // waits for K-half h of the head's weights
        auto w_ready = [&](int h) {
          if (!mbar_wait_bounded(bar(B_W_FULL + h), n & 1, p.err, abort_flag, wait_site(kSitePreWs, 1, 7))) return false;
          tc_fence_after();
          return true;
        };
        const uint32_t l_lo = desc_lo(smem_desc_sw128(sbase + OFF_LAT + x * LAT_SLOT, 16, 1024));
        if (i == 0) {
          if (kt >= 1 && !mbar_wait_bounded(bar(B_ACK_FREE), (kt - 1) & 1, p.err, abort_flag,
                                            wait_site(kSitePreWs, 1, 8))) {
            ok = false;
            break;
          }
          tc_fence_after();
          // ACK = [k~ (1.5 I)] + s_K (1.5 W_K)^T; S = k~ (-3G I) when the before-conv mean is on. The
          // MMAs that read the latent tile go first, so that its slot is released as soon as they are
          // done and the next head's copy can land while the channel mix runs.
          if (pre) {
#pragma unroll
            for (int j = 0; j < D / 16; ++j)
              if (elect_one_sync()) umma_ss_lohi(tmem + T_ACK + 16 * j, l_lo + koff(j), hi, idt_lo[1], hi, id16, 0);
#pragma unroll
            for (int j = 0; j < D / 16; ++j)
              if (elect_one_sync()) umma_ss_lohi(tmem + T_S + 16 * j, l_lo + koff(j), hi, idt_lo[2], hi, id16, 0);
            s_init = true;
          }
          if (elect_one_sync()) umma_commit(bar(B_LAT_FREE + x));
          for (int h = 0; h < 2; ++h) {
            if (!w_ready(h)) {
              ok = false;
              break;
            }
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int kk = 4 * h + k4;
              if (elect_one_sync())
                umma_ss_lohi(tmem + T_ACK, s_lo + koff(kk), hi, w_lo + koff(kk), hi, id128, (pre || kk > 0) ? 1 : 0);
            }
            if (elect_one_sync()) umma_commit(bar(B_W_FREE + h));
          }
          if (!ok) break;
          if (elect_one_sync()) {
            umma_commit(bar(B_S_FREE + x));
            umma_commit(bar(B_ACK_FULL));
          }
        } else {
          const int jq = kt * G + i - 1, y = jq & 1;
          if (jq >= 2 && !mbar_wait_bounded(bar(B_ACQ_FREE + y), ((jq >> 1) & 1) ^ 1, p.err, abort_flag,
                                            wait_site(kSitePreWs, 1, 9))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dq = tmem + T_ACQ + 128 * y;
          // ACQ = [q~_h (0.5 I)] + s_h (1.5 W_h)^T; S += [q~_h (1.5 I)] + s_h (1.5 W_h)^T, the latent
          // tile's MMAs first
          if (pre) {
#pragma unroll
            for (int j = 0; j < D / 16; ++j)
              if (elect_one_sync()) umma_ss_lohi(dq + 16 * j, l_lo + koff(j), hi, idt_lo[0], hi, id16, 0);
#pragma unroll
            for (int j = 0; j < D / 16; ++j)
              if (elect_one_sync()) umma_ss_lohi(tmem + T_S + 16 * j, l_lo + koff(j), hi, idt_lo[1], hi, id16, s_init ? 1 : 0);
            s_init = true;
          }
          if (elect_one_sync()) umma_commit(bar(B_LAT_FREE + x));
          for (int h = 0; h < 2; ++h) {
            if (!w_ready(h)) {
              ok = false;
              break;
            }
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int kk = 4 * h + k4;
              if (elect_one_sync()) umma_ss_lohi(dq, s_lo + koff(kk), hi, w_lo + koff(kk), hi, id128, (pre || kk > 0) ? 1 : 0);
            }
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int kk = 4 * h + k4;
              if (elect_one_sync())
                umma_ss_lohi(tmem + T_S, s_lo + koff(kk), hi, w_lo + koff(kk), hi, id128, (s_init || kk > 0) ? 1 : 0);
            }
            if (elect_one_sync()) umma_commit(bar(B_W_FREE + h));
          }
          if (!ok) break;
          s_init = true;
          if (elect_one_sync()) {
            umma_commit(bar(B_S_FREE + x));
            umma_commit(bar(B_ACQ_FULL + y));
          }
        }
        __syncwarp();
      }
    }
  } else if (warp == W_STORE) {
    // ------------------------------------------------------------------ storer --
    if (lane == 0) {
      prefetch_tmap(&maps.q);
      prefetch_tmap(&maps.ka);
      prefetch_tmap(&maps.kc);
    }
    int stg[2] = {0, 0};
    int kt = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.ntiles && ok; u += gridDim.x, ++kt) {
      const TileId tl = tile_of(p, u);
      // the K head stages nothing in its s slot: its share of that slot's release is given at the
      // first tile, and for later tiles as soon as the previous tile's query heads are stored
      if (kt == 0 && lane == 0) mbar_arrive(bar(B_S_FREE + 0));
      for (int i = 1; i < H1; ++i) {
        const int n = kt * H1 + i, x = n & 1;
        if (!mbar_wait_bounded(bar(B_STAGED + x), stg[x] & 1, p.err, abort_flag, wait_site(kSitePreWs, 2, 10))) {
          ok = false;
          break;
        }
        ++stg[x];
        if (lane == 0) {
          const int h = tl.g * G + i - 1;
          for (int hf = 0; hf < 2; ++hf)
            tma_store_3d(&maps.q, sbase + OFF_SB + x * TILE + hf * HALF, h * D + 64 * hf, tl.t0, tl.b);
          bulk_commit();
          bulk_wait_read<0>();
          mbar_arrive(bar(B_S_FREE + x));
        }
        __syncwarp();
      }
      if (!ok) break;
      if (u + (int)gridDim.x < p.ntiles && lane == 0) mbar_arrive(bar(B_S_FREE + (((kt + 1) * H1) & 1)));
      // the K head: fp16 attention copy, then the bf16 cache, both staged in O
      for (int m = 0; m < 2; ++m) {
        if (!mbar_wait_bounded(bar(B_O_STAGED), (uint32_t)m, p.err, abort_flag, wait_site(kSitePreWs, 2, 11))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          for (int hf = 0; hf < 2; ++hf)
            tma_store_3d(m == 0 ? &maps.ka : &maps.kc, sbase + OFF_O + hf * HALF, tl.g * D + 64 * hf, tl.t0, tl.b);
          bulk_commit();
          bulk_wait_read<0>();
          mbar_arrive(bar(B_O_FREE));
        }
        __syncwarp();
      }
    }
    if (lane == 0) bulk_wait_all();
  } else if (warp < W_EPI0) {
    // -------------------------------------------------------------------- conv --
    const int tc = (warp - W_CONV0) * 32 + lane;  // thread index within the conv warps
    int kt = 0;
    bool ok = true;
    if (p.zero_cnt != nullptr && blockIdx.x == 0)
      for (int i = tc; i < kAttnSplitCounters; i += 128) p.zero_cnt[i] = 0;
    for (int u = blockIdx.x; u < p.ntiles && ok; u += gridDim.x, ++kt) {
      const TileId tl = tile_of(p, u);
      const int tb = kt & 1;
      if (!mbar_wait_bounded(bar(B_TAPS_FULL + tb), (kt >> 1) & 1, p.err, abort_flag, wait_site(kSitePreWs, 3, 12)))
        break;
      const __nv_bfloat16* taps = reinterpret_cast<const __nv_bfloat16*>(smem + OFF_TAPS + tb * TAPS);
      for (int i = 0; i < H1; ++i) {
        const int n = kt * H1 + i, x = n & 1;
        if (!mbar_wait_bounded(bar(B_LAT_FULL + x), (n >> 1) & 1, p.err, abort_flag, wait_site(kSitePreWs, 3, 13)) ||
            (n >= 2 && !mbar_wait_bounded(bar(B_S_FREE + x), ((n >> 1) & 1) ^ 1, p.err, abort_flag,
                                          wait_site(kSitePreWs, 3, 14)))) {
          ok = false;
          break;
        }
        const uint8_t* lat = smem + OFF_LAT + x * LAT_SLOT;
        seq_conv_chunk<KC>(lat, lat + TILE, smem + OFF_SB + x * TILE, taps + (size_t)i * D * K, K, tc & 15, tc >> 4);
        fence_async_smem();  // s, written by threads, is read by the tensor cores
        mbar_arrive(bar(B_S_FULL + x));
      }
      if (!ok) break;
      mbar_arrive(bar(B_TAPS_FREE + tb));
      if (p.v_done) continue;
      // value shift of the group's V head: channels [vfrom, Lkv) of the latent come from the
      // previous token (zero at a sequence start); 8-channel vectors never straddle that boundary
      constexpr int VPER = TT * (D / 8) / 128;
      const long long rowbase = (long long)tl.b * p.S;
      uint4 vsrc[VPER];
#pragma unroll
      for (int k = 0; k < VPER; ++k) {
        const int e = tc + k * 128, rr = e >> 4, vv = e & 15;
        const int t = tl.t0 + rr, gc = tl.g * D + vv * 8;
        const int src = (p.vshift && gc >= p.vfrom) ? t - 1 : t;
        vsrc[k] = make_uint4(0, 0, 0, 0);
        if (t < p.S && src >= 0)
          vsrc[k] = *reinterpret_cast<const uint4*>(p.lat + (rowbase + src) * Nlat + Lq + Lkv + gc);
      }
#pragma unroll
      for (int k = 0; k < VPER; ++k) {
        const int e = tc + k * 128, rr = e >> 4, vv = e & 15;
        const int t = tl.t0 + rr, gc = tl.g * D + vv * 8;
        if (t >= p.S) continue;
        const __half2* h2 = reinterpret_cast<const __half2*>(&vsrc[k]);
        uint32_t hb[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __half22float2(h2[q]);
          hb[q] = pack_bf16x2(f.x, f.y);
        }
        const long long off = (rowbase + t) * Lkv + gc;
        *reinterpret_cast<uint4*>(p.v_cache + off) = make_uint4(hb[0], hb[1], hb[2], hb[3]);
        *reinterpret_cast<uint4*>(p.v_att + off) = vsrc[k];
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue --
    const int quad = warp & 3;                // this warp may touch TMEM lanes [32 quad, 32 quad + 32)
    const int r = quad * 32 + lane;           // token row of the tile
    const int ph = (warp - W_EPI0) >> 2;      // RoPE pairs [32 ph, 32 ph + 32): columns i and i + 64
    const int te = (warp - W_EPI0) * 32 + lane;  // thread index within the epilogue warps
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    bool bad = false;
    float amax = 0.f;
    // side job while the first tile's heads load: this CTA's slice of the W_o fp16 copy
    {
      const long long nvec = p.wo_n / 8;
      const long long chunk = (nvec + gridDim.x - 1) / gridDim.x;
      const long long lo = blockIdx.x * chunk, hi2 = lo + chunk < nvec ? lo + chunk : nvec;
      for (long long e0 = lo + te; e0 < hi2; e0 += 2 * NEPI) {  // two independent loads in flight
        uint4 raw[2];
#pragma unroll
        for (int k = 0; k < 2; ++k)
          if (e0 + k * NEPI < hi2) raw[k] = *reinterpret_cast<const uint4*>(p.wo + (e0 + k * NEPI) * 8);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          if (e0 + k * NEPI >= hi2) continue;
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw[k]);
          uint32_t h[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(b2[q]);
            bad |= f16_overflow(f.x) || f16_overflow(f.y);
            h[q] = pack_f16x2(f.x, f.y);
          }
          *reinterpret_cast<uint4*>(p.wo_lat + (e0 + k * NEPI) * 8) = make_uint4(h[0], h[1], h[2], h[3]);
        }
      }
    }
    const float inv3 = 1.0f / 3.0f, inv3g = 1.0f / (3.0f * (float)G);
    // combine the 8 pairs p0 .. p0 + 7 of this thread (columns p0.. and 64 + p0..) from two
    // tensor-memory column blocks: x = a + b * f, then RoPE; o0 / o1: fp16 of the two column runs
    float cs[32], sn[32];  // RoPE (cos, sin) of this row's 32 pairs, for every head of the tile
    auto combine8 = [&](int k8, const uint32_t* a0, const uint32_t* a1, const uint32_t* b0, const uint32_t* b1,
                        float f, float* v0, float* v1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float x1 = fmaf(u2f(b0[e]), f, u2f(a0[e]));
        const float x2 = fmaf(u2f(b1[e]), f, u2f(a1[e]));
        const float c = cs[8 * k8 + e], sv = sn[8 * k8 + e];
        v0[e] = x1 * c - x2 * sv;
        v1[e] = x2 * c + x1 * sv;
        amax = fmaxf(amax, fmaxf(fabsf(v0[e]), fabsf(v1[e])));
      }
    };
    auto stage8 = [&](uint8_t* stage, int p0, const uint32_t* o0, const uint32_t* o1) {
      const int c0 = p0 / 8;  // chunk c0 of half 0 and of half 1
      *reinterpret_cast<uint4*>(stage + chunk_off(r, c0)) = make_uint4(o0[0], o0[1], o0[2], o0[3]);
      *reinterpret_cast<uint4*>(stage + chunk_off(r, 8 + c0)) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
    };
    int kt = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.ntiles && ok; u += gridDim.x, ++kt) {
      const int tb = kt & 1;
      if (!mbar_wait_bounded(bar(B_RTAB_FULL + tb), (kt >> 1) & 1, p.err, abort_flag, wait_site(kSitePreWs, 4, 15)))
        break;
      // RoPE factors of this row's pairs: angle (t0 + r) theta_i = t0 theta_i (table, reduced in fp64)
      // + r theta_i (fp32: r < 128 keeps the angle to a few ulp)
      {
        const float2* rt = rtab + tb * 64;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const int i = 32 * ph + k;
          float c = 1.f, sv = 0.f;
          if (p.use_rope) {
            const float a = (float)r * thf[i];
            const float kk = rintf(a * 0.15915494f);
            float xr = fmaf(-kk, 6.28318548f, a);  // 2 pi = 6.28318548f - 1.7484555e-7f
            xr = fmaf(kk, 1.7484555e-7f, xr);
            float ca, sa;
            __sincosf(xr, &sa, &ca);
            const float2 t = rt[i];
            c = t.x * ca - t.y * sa;
            sv = t.y * ca + t.x * sa;
          }
          cs[k] = c;
          sn[k] = sv;
        }
      }
      mbar_arrive(bar(B_RTAB_FREE + tb));  // the table is in registers now
      // ---- the query heads: q = ACQ + ACK / 3, RoPE, staged as fp16 in the head's s slot
      for (int j = 0; j < G && ok; ++j) {
        const int jq = kt * G + j, y = jq & 1, x = (kt * H1 + 1 + j) & 1;
        if (!mbar_wait_bounded(bar(B_ACQ_FULL + y), (jq >> 1) & 1, p.err, abort_flag, wait_site(kSitePreWs, 4, 16)) ||
            (j == 0 && !mbar_wait_bounded(bar(B_ACK_FULL), kt & 1, p.err, abort_flag, wait_site(kSitePreWs, 4, 17)))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t aq = lane_addr + T_ACQ + 128 * y;
#pragma unroll
        for (int k8 = 0; k8 < 4; ++k8) {
          const int p0 = 32 * ph + 8 * k8;
          uint32_t a0[8], a1[8], b0[8], b1[8];
          tmem_ld_x8(aq + p0, a0);
          tmem_ld_x8(aq + 64 + p0, a1);
          tmem_ld_x8(lane_addr + T_ACK + p0, b0);
          tmem_ld_x8(lane_addr + T_ACK + 64 + p0, b1);
          tmem_ld_wait();
          float v0[8], v1[8];
          combine8(k8, a0, a1, b0, b1, inv3, v0, v1);
          uint32_t o0[4], o1[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            o0[e] = pack_f16x2(v0[2 * e], v0[2 * e + 1]);
            o1[e] = pack_f16x2(v1[2 * e], v1[2 * e + 1]);
          }
          stage8(smem + OFF_SB + x * TILE, p0, o0, o1);
        }
        // the last query head's ACQ buffer is released after the K head's bf16 values have passed
        // through it
        if (j + 1 < G) {
          tc_fence_before();
          mbar_arrive(bar(B_ACQ_FREE + y));
        }
        fence_async_smem();
        mbar_arrive(bar(B_STAGED + x));
      }
      if (!ok) break;
      // ---- the K head: k = ACK + S / (3G), RoPE; fp16 attention copy staged in O, bf16 cache values
      // parked in this row's columns of the last query head's ACQ buffer
      const int ylast = (kt * G + G - 1) & 1;
      const uint32_t park = lane_addr + T_ACQ + 128 * ylast + 32 * ph;
      uint8_t* kstage = smem + OFF_O;
      if (kt >= 1 &&  // the previous tile's bf16 cache has left O
          !mbar_wait_bounded(bar(B_O_FREE), 1, p.err, abort_flag, wait_site(kSitePreWs, 4, 18)))
        break;
#pragma unroll
      for (int k8 = 0; k8 < 4; ++k8) {
        const int p0 = 32 * ph + 8 * k8;
        uint32_t a0[8], a1[8], b0[8], b1[8];
        tmem_ld_x8(lane_addr + T_ACK + p0, a0);
        tmem_ld_x8(lane_addr + T_ACK + 64 + p0, a1);
        tmem_ld_x8(lane_addr + T_S + p0, b0);
        tmem_ld_x8(lane_addr + T_S + 64 + p0, b1);
        tmem_ld_wait();
        float v0[8], v1[8];
        combine8(k8, a0, a1, b0, b1, inv3g, v0, v1);
        uint32_t o0[4], o1[4], bf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          o0[e] = pack_f16x2(v0[2 * e], v0[2 * e + 1]);
          o1[e] = pack_f16x2(v1[2 * e], v1[2 * e + 1]);
          bf[e] = pack_bf16x2(v0[2 * e], v0[2 * e + 1]);
          bf[4 + e] = pack_bf16x2(v1[2 * e], v1[2 * e + 1]);
        }
        tmem_st_x8(park + 8 * k8, bf);
        stage8(kstage, p0, o0, o1);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_ACK_FREE));  // ACK and S are read: the next tile's K head may overwrite them
      fence_async_smem();
      mbar_arrive(bar(B_O_STAGED));  // the fp16 copy
      if (!mbar_wait_bounded(bar(B_O_FREE), 0, p.err, abort_flag, wait_site(kSitePreWs, 4, 19))) break;
#pragma unroll
      for (int k8 = 0; k8 < 4; ++k8) {
        uint32_t bf[8];
        tmem_ld_x8(park + 8 * k8, bf);
        tmem_ld_wait();
        stage8(kstage, 32 * ph + 8 * k8, bf, bf + 4);
      }
      tc_fence_before();
      mbar_arrive(bar(B_ACQ_FREE + ylast));
      fence_async_smem();
      mbar_arrive(bar(B_O_STAGED));  // the bf16 cache
    }
    // q and k leave as fp16: any value beyond fp16's range (infinities included) is reported
    report_range(bad || amax > 65504.0f, p.err);
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) spin_ns(20000ull);  // copies or MMAs issued before a timed-out wait may still land
  tc_fence_after();
  if (warp == W_MMA) tmem_dealloc(tmem, 512);
}

bool encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* ptr, const cuuint64_t* dims,
            const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn enc = get_encode_tiled();
  if (enc == nullptr) return false;
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, dt, (cuuint32_t)rank, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D map [B][S][width] of 16-bit elements, box 64 x rows x 1
bool encode_bsw(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, int B, int S, int width, int rows) {
  const cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)S, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)width * 2, (cuuint64_t)width * S * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  return encode(m, dt, 3, ptr, dims, strides, box);
}

}  // namespace

bool preproc_ws_supported(const BlockDims& dm) {
  return dm.io == DType::BF16 && dm.lat == DType::F16 && dm.d == D && dm.K >= 1 && dm.K <= KMAX && dm.G >= 1 &&
         dm.G <= GMAX && (dm.qk_mean_mode & 2) != 0 && smem_bytes(dm.G + 1, dm.K) <= kSmemLimit &&
         ((long long)dm.E * dm.Lq) % 8 == 0;
}

cudaError_t launch_preproc_ws(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream) {
  if (!preproc_ws_supported(dm) || p.wc_lat == nullptr) return cudaErrorInvalidValue;
  WsMaps maps;
  const CUtensorMapDataType f16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16, bf16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!encode_bsw(&maps.lat, f16, p.qkv_lat, dm.B, dm.S, dm.Nlat, TT) ||
      !encode_bsw(&maps.halo, f16, p.qkv_lat, dm.B, dm.S, dm.Nlat, dm.K > 1 ? dm.K - 1 : 1) ||
      !encode_bsw(&maps.q, f16, p.q, dm.B, dm.S, dm.Lq, TT) ||
      !encode_bsw(&maps.ka, f16, p.k_att, dm.B, dm.S, dm.Lkv, TT) ||
      !encode_bsw(&maps.kc, bf16, p.k_cache, dm.B, dm.S, dm.Lkv, TT))
    return cudaErrorInvalidValue;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)(dm.nq + dm.nkv) * D};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 128};
    if (!encode(&maps.wc, f16, 2, p.wc_lat, dims, strides, box)) return cudaErrorInvalidValue;
  }
  WsParams q;
  q.lat = static_cast<const __half*>(p.qkv_lat);
  q.q = static_cast<__half*>(p.q);
  q.cq_seq = static_cast<const __nv_bfloat16*>(p.cq_seq);
  q.ck_seq = static_cast<const __nv_bfloat16*>(p.ck_seq);
  q.v_cache = static_cast<__nv_bfloat16*>(p.v_cache);
  q.v_att = static_cast<__half*>(p.v_att);
  q.wo = static_cast<const __nv_bfloat16*>(p.Wo);
  q.wo_lat = static_cast<__half*>(p.wo_lat);
  q.wo_n = (long long)dm.E * dm.Lq;
  q.err = p.dev_err;
  q.zero_cnt = attention_tc_supported(dm) ? static_cast<int*>(p.sched) : nullptr;
  q.B = dm.B;
  q.S = dm.S;
  q.nq = dm.nq;
  q.nkv = dm.nkv;
  q.K = dm.K;
  q.pre = dm.qk_mean_mode & 1;
  q.vshift = dm.value_shift;
  q.vfrom = dm.vshift_from;
  q.use_rope = dm.use_rope;
  q.v_done = p.v_fused ? 1 : 0;
  q.nT = (dm.S + TT - 1) / TT;
  q.ntiles = dm.B * q.nT * dm.nkv;
  Theta th;
  for (int i = 0; i < D / 2; ++i) th.v[i] = pow((double)dm.rope_base, -2.0 * (double)i / (double)D);
  const int smem = smem_bytes(dm.G + 1, dm.K);
  const int grid = q.ntiles < num_sms() ? q.ntiles : num_sms();
  cudaError_t e;
  if (dm.K == 4) {
    if ((e = cudaFuncSetAttribute(preproc_ws_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return e;
    preproc_ws_kernel<4><<<grid, NT, smem, stream>>>(maps, q, th);
  } else {
    if ((e = cudaFuncSetAttribute(preproc_ws_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return e;
    preproc_ws_kernel<0><<<grid, NT, smem, stream>>>(maps, q, th);
  }
  return cudaGetLastError();
}

}  // namespace cca
