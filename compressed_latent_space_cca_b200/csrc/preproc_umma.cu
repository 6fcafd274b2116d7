// Latent preprocessing of one CCA / CCGQA block (steps a2-a8: seq conv, channel conv, QK-mean
// before and after, RoPE, value shift, KV-cache write) for bf16 blocks with head_dim 128, in a
// tensor-memory form: the channel mix runs as tcgen05 MMAs and every per-token step reads its
// operands from TMEM, one thread per token row.
//
// "Compressed Convolutional Attention" (gist.science/es/paper/2510.04476), section 2.B items 1-3
// and section 3 item 2; the forms follow the same readings as the mma.sync kernel (depthwise
// causal seq conv with tap K-1 on the current token, per-head dense channel mix, both QK-mean
// terms added to the conv outputs, rotate-half RoPE, upper half of the V latent shifted by one
// token).
//
// One CTA = 128 tokens of one sequence x one KV group, 8 warps. For each head of the group (the K
// head first, then the G query heads):
//   - the head's fp16 latents (128 tokens plus a K-1 token halo) arrive by TMA through a 3D map
//     [B][S][Nlat], so halo rows before a sequence start read as zeros (128-byte swizzle); the
//     next head's latents and channel weights load while the current head is processed;
//   - the causal seq conv runs on CUDA cores in fp32 and its output s is rounded to fp16 straight
//     into the K-major, 128-byte-swizzled layout of a tcgen05 A operand;
//   - one elected lane issues the 8 MMAs (M128 N128 K16, fp16, fp32 accumulate) of c = s W_c^T;
//     query heads also accumulate into a second block of columns that ends up holding the sum of
//     the c_q over the group;
//   - query heads: thread r (TMEM lane r) combines c_q, c_k and the raw latents of its token,
//     applies RoPE to its pairs (i, i+64), adds its raw q~ into the running sum kept in TMEM, and
//     stages q in shared memory for a TMA tensor store.
// Then the K head's combine and RoPE with the group sums, staged as the bf16 cache and the fp16
// attention copy (two TMA stores), and the value shift with 16-byte loads and stores.
//
// Tensor memory (512 columns): c_k | sum of c_q | current c_q | sum of raw q~.
// Every mbarrier wait is bounded; on expiry the CTA records the wait site, stops, gives copies and
// MMAs in flight a bounded 20 us to land and releases its tensor memory.
#include <math.h>

#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

constexpr int D = 128;
constexpr int TT = 128;        // tokens per CTA (one TMEM lane each)
constexpr int NT = 256;        // threads
constexpr int KMAX = 8;        // largest seq-conv kernel of this path
constexpr int GMAX = 8;        // largest group of this path
constexpr int ZRMAX = TT + KMAX - 1;
constexpr int ZHALF = 17 * 1024;         // one 64-column half of a head's latents: up to 136 rows of 128 B
constexpr int ZHEAD = 2 * ZHALF;         // one head's staged latents
constexpr int TILE = TT * D * 2;         // a 128 x 128 16-bit tile (two 64-column halves of 16 KB)
constexpr int HALF = TILE / 2;
constexpr uint32_t ACK = 0, ACS = 128, ACQ = 256, AQS = 384;  // TMEM column blocks

// shared memory: [LK][LQ0][LQ1][SB][WB0][WB1][taps][rtab][barriers]
constexpr int OFF_LK = 0;
constexpr int OFF_LQ = OFF_LK + ZHEAD;
constexpr int OFF_SB = OFF_LQ + 2 * ZHEAD;
constexpr int OFF_WB = OFF_SB + TILE;
constexpr int OFF_TAPS = OFF_WB + 2 * TILE;
constexpr int TAPS_BYTES = (GMAX + 1) * D * KMAX * 2;
constexpr int OFF_RTAB = OFF_TAPS + TAPS_BYTES;
constexpr int OFF_THF = OFF_RTAB + (D / 2) * 8;
constexpr int OFF_BAR = OFF_THF + (D / 2) * 4;
constexpr int SMEM_BYTES = OFF_BAR + 128 + 1024;  // barriers, TMEM slot, abort flag; alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory of one CTA");
static_assert(ZRMAX * 128 <= ZHALF, "latent half");

struct Theta {
  double v[D / 2];  // base^(-2i/d)
};

struct UmmaMaps {
  CUtensorMap lat;  // [B][S][Nlat] fp16, box 64 x (TT+K-1) x 1
  CUtensorMap wc;   // [(nq+nkv)*D][D] fp16 channel weights, box 64 x 128
  CUtensorMap q;    // [B][S][Lq] fp16, box 64 x 128 x 1 (store)
  CUtensorMap kc;   // [B][S][Lkv] bf16 K cache (store)
  CUtensorMap ka;   // [B][S][Lkv] fp16 attention copy of k (store)
};

struct UmmaParams {
  const __half* lat;  // [T, Nlat] (value shift reads)
  const __nv_bfloat16 *cq_seq, *ck_seq;
  __nv_bfloat16* v_cache;  // [T, Lkv]
  __half* v_att;           // [T, Lkv]
  const __nv_bfloat16* wo;  // [E, Lq] (fp16 copy made here as a side job)
  __half* wo_lat;
  long long wo_n;
  unsigned* err;
  int* zero_cnt;  // split-pair counters of the attention launch that follows (cleared here)
  int S, nq, nkv, K, mode, vshift, use_rope;
};

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32"
      " [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Byte offset of 16-bit element (row, col) of a 128-column tile stored as two 64-column halves of
// 128-byte rows with the 128-byte swizzle (16-byte chunk c of row r at position c ^ (r % 8)): the
// layout of a TMA box with SWIZZLE_128B and of a K-major tcgen05 operand.
__device__ __forceinline__ uint32_t sw128(int row, int col, int half_bytes) {
  const int h = col >> 6, c = (col >> 3) & 7, w = col & 7;
  return (uint32_t)(h * half_bytes + row * 128 + (((c ^ (row & 7)) << 4) | (w << 1)));
}

// Spins for about `ns` nanoseconds (a bounded drain after an abort).
__device__ __forceinline__ void spin_ns(unsigned long long ns) {
  const unsigned long long t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 < ns) {
  }
}

__global__ void __launch_bounds__(NT, 1) preproc_umma_kernel(const __grid_constant__ UmmaMaps maps,
                                                            const __grid_constant__ UmmaParams p,
                                                            const __grid_constant__ Theta th) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  __nv_bfloat16* taps = reinterpret_cast<__nv_bfloat16*>(smem + OFF_TAPS);  // [H1][D][K]
  float2* rtab = reinterpret_cast<float2*>(smem + OFF_RTAB);                 // (cos, sin) of t0 theta_i
  float* thf = reinterpret_cast<float*>(smem + OFF_THF);                      // theta_i in fp32
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* lat_bar = bars;      // [3]: K head latents, query-head buffers 0 and 1
  uint64_t* w_bar = bars + 3;    // [2]: weight buffers
  uint64_t* acc_bar = bars + 5;  // MMAs of the current head done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int G = p.nq / p.nkv, H1 = G + 1, KK = p.K, ZR = TT + KK - 1;
  const int Lq = p.nq * D, Lkv = p.nkv * D, Nlat = Lq + 2 * Lkv;
  const int t0 = blockIdx.x * TT, g = blockIdx.y, b = blockIdx.z;
  const long long rowbase = (long long)b * p.S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lat_bytes = 2u * (uint32_t)ZR * 128u;
  bool bad = false;
  float amax = 0.f;

  // latent columns and channel-weight rows of head i of the group (0: the K head, i >= 1: query
  // head i - 1)
  auto lat_col = [&](int i) { return i == 0 ? Lq + g * D : (g * G + i - 1) * D; };
  auto wc_row = [&](int i) { return i == 0 ? (p.nq + g) * D : (g * G + i - 1) * D; };
  auto lat_buf = [&](int i) { return i == 0 ? OFF_LK : OFF_LQ + ((i - 1) & 1) * ZHEAD; };
  auto lat_barrier = [&](int i) { return smem_u32(&lat_bar[i == 0 ? 0 : 1 + ((i - 1) & 1)]); };
  // thread 0 issues the copies of head i: latents and channel weights
  auto issue_loads = [&](int i) {
    const uint32_t lb = lat_barrier(i), wb = smem_u32(&w_bar[i & 1]);
    mbar_arrive_expect_tx(lb, lat_bytes);
    for (int h = 0; h < 2; ++h)
      tma_load_3d(sbase + lat_buf(i) + h * ZHALF, &maps.lat, lb, lat_col(i) + 64 * h, t0 - (KK - 1), b);
    mbar_arrive_expect_tx(wb, TILE);
    for (int h = 0; h < 2; ++h)
      tma_load_2d(sbase + OFF_WB + (i & 1) * TILE + h * HALF, &maps.wc, wb, 64 * h, wc_row(i));
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(smem_u32(&lat_bar[i]), 1);
    for (int i = 0; i < 2; ++i) mbar_init(smem_u32(&w_bar[i]), 1);
    mbar_init(smem_u32(acc_bar), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    prefetch_tmap(&maps.lat);
    prefetch_tmap(&maps.wc);
    issue_loads(0);
  }

  // seq-conv taps of the group's heads, [H1][D][K] in processing order (K head first): the K
  // head's D*K taps, then the G query heads' (contiguous in cq_seq); 16-byte vectors when both
  // sources allow them (D*K is a multiple of 8), every load issued before the stores
  {
    const __nv_bfloat16* qs = p.cq_seq + (long long)g * G * D * KK;
    const __nv_bfloat16* ks = p.ck_seq + (long long)g * D * KK;
    const int nk8 = D * KK / 8, n8 = H1 * D * KK / 8;
    if (((reinterpret_cast<uintptr_t>(qs) | reinterpret_cast<uintptr_t>(ks)) & 15) == 0) {
      constexpr int PER = ((GMAX + 1) * D * KMAX / 8 + NT - 1) / NT;
      uint4 v[PER];
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int e = threadIdx.x + k * NT;
        if (e < n8)
          v[k] = e < nk8 ? reinterpret_cast<const uint4*>(ks)[e] : reinterpret_cast<const uint4*>(qs)[e - nk8];
      }
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int e = threadIdx.x + k * NT;
        if (e < n8) reinterpret_cast<uint4*>(taps)[e] = v[k];
      }
    } else {
      for (int e = threadIdx.x; e < H1 * D * KK; e += NT)
        taps[e] = e < D * KK ? ks[e] : qs[e - D * KK];
    }
  }
  // RoPE table: (cos, sin) of t0 * theta_i, the angle reduced modulo 2 pi in fp64
  if (p.use_rope && threadIdx.x < D / 2) {
    const int i = threadIdx.x;
    const double a = (double)t0 * th.v[i];
    const double k = rint(a * 0.15915494309189535);
    double r = fma(-k, 6.283185307179586, a);
    r = fma(-k, 2.4492935982947064e-16, r);
    float c, sn;
    sincosf((float)r, &sn, &c);
    rtab[i] = make_float2(c, sn);
    thf[i] = (float)th.v[i];
  }
  // side jobs while the first copies are in flight: this CTA's slice of the W_o fp16 copy, and the
  // attention's split counters
  {
    const long long nvec = p.wo_n / 8;
    const long long nct = (long long)gridDim.x * gridDim.y * gridDim.z;
    const long long cid = ((long long)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    const long long chunk = (nvec + nct - 1) / nct;
    const long long lo = cid * chunk, hi = lo + chunk < nvec ? lo + chunk : nvec;
    for (long long e0 = lo + threadIdx.x; e0 < hi; e0 += 4 * NT) {  // four independent loads in flight
      uint4 raw[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (e0 + k * NT < hi) raw[k] = *reinterpret_cast<const uint4*>(p.wo + (e0 + k * NT) * 8);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (e0 + k * NT >= hi) continue;
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw[k]);
        uint32_t h[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __bfloat1622float2(b2[q]);
          bad |= f16_overflow(f.x) || f16_overflow(f.y);
          h[q] = pack_f16x2(f.x, f.y);
        }
        *reinterpret_cast<uint4*>(p.wo_lat + (e0 + k * NT) * 8) = make_uint4(h[0], h[1], h[2], h[3]);
      }
    }
    if (p.zero_cnt != nullptr && cid == 0)
      for (int i = threadIdx.x; i < kAttnSplitCounters; i += NT) p.zero_cnt[i] = 0;
  }
  __syncthreads();

  // epilogue geometry: thread = token row r (TMEM lane), pairs [32 cg, 32 cg + 32) and their partners
  const int quad = warp & 3, cg = warp >> 2;
  const int r = quad * 32 + lane;
  const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
  const int zrow = r + KK - 1;  // the token's own row in the staged latents
  // RoPE factors of a pair: angle (t0 + r) theta_i = t0 theta_i (table) + r theta_i (fp32, < 128 rad)
  auto rope_cs = [&](int i, float& c, float& s) {
    c = 1.f;
    s = 0.f;
    if (!p.use_rope) return;
    const float a = (float)r * thf[i];  // r < 128: fp32 keeps the angle to a few ulp
    const float k = rintf(a * 0.15915494f);
    float x = fmaf(-k, 6.28318548f, a);  // 2 pi = 6.28318548f - 1.7484555e-7f
    x = fmaf(k, 1.7484555e-7f, x);
    float ca, sa;
    __sincosf(x, &sa, &ca);
    const float2 t = rtab[i];
    c = t.x * ca - t.y * sa;
    s = t.y * ca + t.x * sa;
  };
  // 8 consecutive fp16 latents of head buffer `buf` at (row, col), as floats
  auto lat8 = [&](int buf, int row, int col, float* out) {
    const uint4 v = *reinterpret_cast<const uint4*>(smem + buf + sw128(row, col, ZHALF));
    const __half2* h2 = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(h2[k]);
      out[2 * k] = f.x;
      out[2 * k + 1] = f.y;
    }
  };

  const uint32_t idesc = idesc_f32acc(128, D, 0, 0, kFmtF16);
  const uint64_t adesc0 = smem_desc_sw128(sbase + OFF_SB, 16, 1024);
  const bool pre = (p.mode & 1) != 0, post = (p.mode & 2) != 0;

  for (int i = 0; i < H1; ++i) {
    // the next head's copies go into the buffers head i - 1 used, which it has finished with
    // (thread 0, which also issues the q stores and so owns their bulk groups: the buffer the next
    // weights go into may still be read by the store of head i - 2's q, staged there)
    if (i + 1 < H1 && threadIdx.x == 0) {
      bulk_wait_read<0>();
      issue_loads(i + 1);
    }
    const int lb = lat_buf(i);
    const uint32_t lpar = i == 0 ? 0u : (uint32_t)(((i - 1) >> 1) & 1);
    if (!mbar_wait_bounded(lat_barrier(i), lpar, p.err, abort_flag, wait_site(kSitePreUmma, 1, 1))) goto done;

    // ---- causal seq conv of head i into s (fp16, tcgen05 A layout): thread = column pair cp,
    // 32 consecutive rows, the last K latent rows in registers
    {
      const int cp = threadIdx.x & 63, rb = (threadIdx.x >> 6) * 32;
      const __nv_bfloat16* w = taps + (size_t)i * D * KK;
      float w0[KMAX], w1[KMAX];
      float wl0 = 0.f, wl1 = 0.f;  // tap K-1, on the current token
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        w0[j] = j < KK ? __bfloat162float(w[(2 * cp) * KK + j]) : 0.f;
        w1[j] = j < KK ? __bfloat162float(w[(2 * cp + 1) * KK + j]) : 0.f;
        if (j == KK - 1) {
          wl0 = w0[j];
          wl1 = w1[j];
        }
      }
      auto zat = [&](int row) {
        return __half22float2(*reinterpret_cast<const __half2*>(smem + lb + sw128(row, 2 * cp, ZHALF)));
      };
      // win[j], j < K-1: staged row rb + t + j (token t - (K-1) + j of output row t = rb + t)
      float2 win[KMAX - 1];
#pragma unroll
      for (int j = 0; j < KMAX - 1; ++j) win[j] = j < KK - 1 ? zat(rb + j) : make_float2(0.f, 0.f);
#pragma unroll 4
      for (int t = 0; t < 32; ++t) {
        const float2 cur = zat(rb + t + KK - 1);
        float a0 = wl0 * cur.x, a1 = wl1 * cur.y;
#pragma unroll
        for (int j = 0; j < KMAX - 1; ++j)
          if (j < KK - 1) {
            a0 = fmaf(w0[j], win[j].x, a0);
            a1 = fmaf(w1[j], win[j].y, a1);
          }
        // slide the window by one row (static indices only)
#pragma unroll
        for (int j = 0; j < KMAX - 1; ++j) {
          if (j + 1 < KMAX - 1 && j + 1 < KK - 1) win[j] = win[j + 1 < KMAX - 1 ? j + 1 : j];
          else if (j == KK - 2) win[j] = cur;
        }
        *reinterpret_cast<__half2*>(smem + OFF_SB + sw128(rb + t, 2 * cp, HALF)) = __floats2half2_rn(a0, a1);
      }
    }
    fence_async_smem();  // s, written by threads, is read by the tensor cores
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- channel mix: c = s W^T into c_k (K head) or c_q, and for query heads into the c_q sum
    if (warp == 0) {
      if (!mbar_wait_bounded(smem_u32(&w_bar[i & 1]), (uint32_t)((i >> 1) & 1), p.err, abort_flag,
                             wait_site(kSitePreUmma, 2, 2)))
        goto mma_skip;
      tc_fence_after();
      {
        const uint64_t bdesc0 = smem_desc_sw128(sbase + OFF_WB + (i & 1) * TILE, 16, 1024);
        const uint32_t a_lo0 = desc_lo(adesc0), b_lo0 = desc_lo(bdesc0), hi = desc_hi(adesc0);
        const int nsum = (i > 0 && post) ? 2 : 1;
        for (int dst = 0; dst < nsum; ++dst) {
          const uint32_t dcol = i == 0 ? ACK : (dst == 0 ? ACQ : ACS);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            // K step kk: half kk / 4 (16 KB apart), 32 bytes per step within the half
            const uint32_t off = (uint32_t)((kk >> 2) * (HALF >> 4) + (kk & 3) * 2);
            const uint32_t acc = (dst == 1 && i > 1) || kk > 0;
            if (elect_one_sync()) umma_ss_lohi(tmem + dcol, a_lo0 + off, hi, b_lo0 + off, hi, idesc, acc);
          }
        }
        if (elect_one_sync()) umma_commit(smem_u32(acc_bar));
      }
    mma_skip:;
    }
    if (!mbar_wait_bounded(smem_u32(acc_bar), (uint32_t)(i & 1), p.err, abort_flag, wait_site(kSitePreUmma, 3, 3)))
      goto done;
    tc_fence_after();

    if (i > 0) {
      // ---- query head i - 1: q = c_q + PRE (q~ + k~)/2 + POST (c_q + c_k)/2, RoPE, staged in the
      // weight buffer this head's MMAs have finished reading (free until the loads of head i + 2),
      // so the next head's conv need not wait for the store
      const int qb = lb;
      const int qstage = OFF_WB + (i & 1) * TILE;
#pragma unroll 1
      for (int sub = 0; sub < 2; ++sub) {
        const int i0 = cg * 32 + sub * 16;  // pairs i0 .. i0 + 15: columns i and i + 64
        uint32_t cq[2][16], ck[2][16], qs[2][16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tmem_ld_x16(lane_addr + ACQ + i0 + 64 * h, cq[h]);
          tmem_ld_x16(lane_addr + ACK + i0 + 64 * h, ck[h]);
          if (pre && i > 1) tmem_ld_x16(lane_addr + AQS + i0 + 64 * h, qs[h]);
        }
        tmem_ld_wait();
        float v[2][16];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c8 = 0; c8 < 2; ++c8) {
            float zq[8], zk[8];
            lat8(qb, zrow, i0 + 64 * h + 8 * c8, zq);
            lat8(OFF_LK, zrow, i0 + 64 * h + 8 * c8, zk);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int k = 8 * c8 + e;
              const float cqv = u2f(cq[h][k]), ckv = u2f(ck[h][k]);
              float x = cqv;
              if (pre) x += 0.5f * (zq[e] + zk[e]);
              if (post) x += 0.5f * (cqv + ckv);
              v[h][k] = x;
              // running sum of the raw q~ over the group's heads (for the K head's PRE term)
              qs[h][k] = __float_as_uint((i > 1 ? u2f(qs[h][k]) : 0.f) + zq[e]);
            }
          }
        if (pre) {
#pragma unroll
          for (int h = 0; h < 2; ++h) tmem_st_x16(lane_addr + AQS + i0 + 64 * h, qs[h]);
          tmem_st_wait();
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          float c, s;
          rope_cs(i0 + k, c, s);
          const float x1 = v[0][k], x2 = v[1][k];
          v[0][k] = x1 * c - x2 * s;
          v[1][k] = x2 * c + x1 * s;
          amax = fmaxf(amax, fmaxf(fabsf(v[0][k]), fabsf(v[1][k])));
        }
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c8 = 0; c8 < 2; ++c8) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) w4[e] = pack_f16x2(v[h][8 * c8 + 2 * e], v[h][8 * c8 + 2 * e + 1]);
            *reinterpret_cast<uint4*>(smem + qstage + sw128(r, i0 + 64 * h + 8 * c8, HALF)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      if (threadIdx.x == 0) {
        const int h = g * G + i - 1;
        for (int hf = 0; hf < 2; ++hf) tma_store_3d(&maps.q, sbase + qstage + hf * HALF, h * D + 64 * hf, t0, b);
        bulk_commit();
      }
      __syncthreads();
    }
  }

  // the K head stages in s and weight buffer 0: the last q store must have read its buffer
  if (threadIdx.x == 0) bulk_wait_read<0>();
  __syncthreads();
  {  // (a block of its own: the waits above leave to `done` past its declarations)
  // value-shift sources, loaded now so that their latency overlaps the K head's combine: channels
  // [Lkv/2, Lkv) come from the previous token (0 at a sequence start); 8-channel vectors never
  // straddle that boundary
  constexpr int VPER = TT * (D / 8) / NT;
  uint4 vsrc[VPER];
#pragma unroll
  for (int k = 0; k < VPER; ++k) {
    const int e = threadIdx.x + k * NT, rr = e / (D / 8), vv = e % (D / 8);
    const int t = t0 + rr, gc = g * D + vv * 8;
    const int src = (p.vshift && gc >= Lkv / 2) ? t - 1 : t;
    vsrc[k] = make_uint4(0, 0, 0, 0);
    if (t < p.S && src >= 0) vsrc[k] = *reinterpret_cast<const uint4*>(p.lat + (rowbase + src) * Nlat + Lq + Lkv + gc);
  }

  // ---- the K head: k = c_k + PRE (mean q~ + k~)/2 + POST (mean c_q + c_k)/2, RoPE; staged as the
  // bf16 cache in s and the fp16 attention copy in weight buffer 0 (every MMA has completed)
  {
    const float invG = 1.f / (float)G;
#pragma unroll 1
    for (int sub = 0; sub < 2; ++sub) {
      const int i0 = cg * 32 + sub * 16;
      uint32_t ck[2][16], cs[2][16], qs[2][16];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tmem_ld_x16(lane_addr + ACK + i0 + 64 * h, ck[h]);
        if (post) tmem_ld_x16(lane_addr + ACS + i0 + 64 * h, cs[h]);
        if (pre) tmem_ld_x16(lane_addr + AQS + i0 + 64 * h, qs[h]);
      }
      tmem_ld_wait();
      float v[2][16];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c8 = 0; c8 < 2; ++c8) {
          float zk[8];
          lat8(OFF_LK, zrow, i0 + 64 * h + 8 * c8, zk);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int k = 8 * c8 + e;
            const float ckv = u2f(ck[h][k]);
            float x = ckv;
            if (pre) x += 0.5f * (u2f(qs[h][k]) * invG + zk[e]);
            if (post) x += 0.5f * (u2f(cs[h][k]) * invG + ckv);
            v[h][k] = x;
          }
        }
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        float c, s;
        rope_cs(i0 + k, c, s);
        const float x1 = v[0][k], x2 = v[1][k];
        v[0][k] = x1 * c - x2 * s;
        v[1][k] = x2 * c + x1 * s;
        amax = fmaxf(amax, fmaxf(fabsf(v[0][k]), fabsf(v[1][k])));
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c8 = 0; c8 < 2; ++c8) {
          uint32_t wb[4], wh[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            wb[e] = pack_bf16x2(v[h][8 * c8 + 2 * e], v[h][8 * c8 + 2 * e + 1]);
            wh[e] = pack_f16x2(v[h][8 * c8 + 2 * e], v[h][8 * c8 + 2 * e + 1]);
          }
          const uint32_t o = sw128(r, i0 + 64 * h + 8 * c8, HALF);
          *reinterpret_cast<uint4*>(smem + OFF_SB + o) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
          *reinterpret_cast<uint4*>(smem + OFF_WB + o) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int hf = 0; hf < 2; ++hf) {
        tma_store_3d(&maps.kc, sbase + OFF_SB + hf * HALF, g * D + 64 * hf, t0, b);
        tma_store_3d(&maps.ka, sbase + OFF_WB + hf * HALF, g * D + 64 * hf, t0, b);
      }
      bulk_commit();
    }
  }

  // ---- value shift: the bf16 cache and the fp16 attention copy of the shifted v
#pragma unroll
  for (int k = 0; k < VPER; ++k) {
    const int e = threadIdx.x + k * NT, rr = e / (D / 8), vv = e % (D / 8);
    const int t = t0 + rr, gc = g * D + vv * 8;
    if (t >= p.S) continue;
    const uint4 hv = vsrc[k];
    const __half2* h2 = reinterpret_cast<const __half2*>(&hv);
    uint32_t hb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(h2[k]);
      hb[k] = pack_bf16x2(f.x, f.y);
    }
    const long long off = (rowbase + t) * Lkv + gc;
    *reinterpret_cast<uint4*>(p.v_cache + off) = make_uint4(hb[0], hb[1], hb[2], hb[3]);
    *reinterpret_cast<uint4*>(p.v_att + off) = hv;
  }
  }

done:
  // q and k leave as fp16: any value beyond fp16's range (infinities included) is reported
  report_range(bad || amax > 65504.0f, p.err);
  if (threadIdx.x == 0) bulk_wait_all();  // the staged stores finish before shared memory goes
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) spin_ns(20000ull);  // copies or MMAs issued before a timed-out wait may still land
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
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

bool preproc_umma_supported(const BlockDims& dm) {
  return dm.io == DType::BF16 && dm.lat == DType::F16 && dm.d == D && dm.K >= 1 && dm.K <= KMAX && dm.G >= 1 &&
         dm.G <= GMAX && ((long long)dm.E * dm.Lq) % 8 == 0;
}

cudaError_t launch_preproc_umma(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream) {
  if (!preproc_umma_supported(dm) || p.wc_lat == nullptr) return cudaErrorInvalidValue;
  UmmaMaps maps;
  const CUtensorMapDataType f16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16, bf16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!encode_bsw(&maps.lat, f16, p.qkv_lat, dm.B, dm.S, dm.Nlat, TT + dm.K - 1) ||
      !encode_bsw(&maps.q, f16, p.q, dm.B, dm.S, dm.Lq, TT) ||
      !encode_bsw(&maps.kc, bf16, p.k_cache, dm.B, dm.S, dm.Lkv, TT) ||
      !encode_bsw(&maps.ka, f16, p.k_att, dm.B, dm.S, dm.Lkv, TT))
    return cudaErrorInvalidValue;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)(dm.nq + dm.nkv) * D};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 128};
    if (!encode(&maps.wc, f16, 2, p.wc_lat, dims, strides, box)) return cudaErrorInvalidValue;
  }
  UmmaParams q;
  q.lat = static_cast<const __half*>(p.qkv_lat);
  q.cq_seq = static_cast<const __nv_bfloat16*>(p.cq_seq);
  q.ck_seq = static_cast<const __nv_bfloat16*>(p.ck_seq);
  q.v_cache = static_cast<__nv_bfloat16*>(p.v_cache);
  q.v_att = static_cast<__half*>(p.v_att);
  q.wo = static_cast<const __nv_bfloat16*>(p.Wo);
  q.wo_lat = static_cast<__half*>(p.wo_lat);
  q.wo_n = (long long)dm.E * dm.Lq;
  q.err = p.dev_err;
  q.zero_cnt = attention_tc_supported(dm) ? static_cast<int*>(p.sched) : nullptr;
  q.S = dm.S;
  q.nq = dm.nq;
  q.nkv = dm.nkv;
  q.K = dm.K;
  q.mode = dm.qk_mean_mode;
  q.vshift = dm.value_shift;
  q.use_rope = dm.use_rope;
  Theta th;
  for (int i = 0; i < D / 2; ++i) th.v[i] = pow((double)dm.rope_base, -2.0 * (double)i / (double)D);
  cudaError_t e = cudaFuncSetAttribute(preproc_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((dm.S + TT - 1) / TT, dm.nkv, dm.B);
  preproc_umma_kernel<<<grid, NT, SMEM_BYTES, stream>>>(maps, q, th);
  return cudaGetLastError();
}

}  // namespace cca
