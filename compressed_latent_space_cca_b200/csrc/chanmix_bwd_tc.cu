// Channel-mix backward of one CCA head on tcgen05, head_dim 128.
//
// "Compressed Convolutional Attention" (gist.science/es/paper/2510.04476, section 2.B item 1: a
// dense d x d mix within each head after the causal sequence conv). With c[t] = W_c s[t] and the
// gradient dc of c:
//   ds[t] = W_c^T dc[t]            (the gradient passed on to the sequence conv)
//   dW_c  = sum_t dc[t] s[t]^T     (s recomputed from the latents by the sequence conv)
// A CTA per (block of rows, head) walks 128-row tiles. W_c arrives by asynchronous 16-byte copies
// straight into its swizzled operand layout, and each tile's dc (fp32) is copied the same way into a
// staging buffer while the previous tile's MMAs and ds rows run. Its 512 threads (a column and a
// quarter of the rows each) read dc from there and the latent rows from global memory, recompute s,
// and write both as bf16 pairs hi = bf16(v), lo = bf16(v - hi) into shared memory (128-byte swizzle). The dc tile serves twice: K-major (rows t,
// k = i) as the A operand of ds, and read MN-major (m = i, k = t) as the A operand of dW_c. One
// elected thread issues the MMAs:
//   ds (TMEM columns 0..127)    = [dc_hi | dc_lo] x [W_c; W_c]       (K = 256 over the two segments)
//   dW_c (TMEM columns 128..255) += dc_hi s_hi^T + dc_hi s_lo^T + dc_lo s_hi^T   (K = t)
// W_c stays in shared memory (bf16, exact) for all tiles; dW_c accumulates in TMEM across them and
// is added to the fp32 sum once per CTA with vector atomics. Every mbarrier wait is bounded.
#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

constexpr int CD = 128;        // head_dim
constexpr int CT = 128;        // rows per tile
constexpr int CT_THREADS = 512;
constexpr int CT_RQ = CT_THREADS / CD;  // row quarters of a tile
constexpr int CT_RROWS = CT / CT_RQ;    // rows of a tile per thread
constexpr int HALF = CT * 128;  // 16 KB: 128 rows x 64 bf16 (one 128-byte swizzle span)
// shared memory: W_c [2 column halves], dc [4 K chunks: hi i 0-63, hi i 64-127, lo, lo],
// s [4: hi j 0-63, hi j 64-127, lo, lo], the next tile's dc (fp32 [128 rows][128]), barrier
constexpr int OFF_W = 0;
constexpr int OFF_DC = OFF_W + 2 * HALF;
constexpr int OFF_S = OFF_DC + 4 * HALF;
constexpr int OFF_STG = OFF_S + 4 * HALF;
constexpr int OFF_BAR = OFF_STG + CT * CD * 4;
constexpr size_t CT_SMEM = OFF_BAR + 64 + 1024;
static_assert(CT_SMEM <= 232448, "shared memory of one CTA");
constexpr int CT_KMAX = 8;

// byte offset of element (row, col) of a [rows][64-column half] bf16 tile with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw_off(int row, int col) {
  return (uint32_t)(row * 128 + ((((col >> 3) ^ (row & 7)) << 4) | ((col & 7) << 1)));
}

__device__ __forceinline__ void st_bf16(uint8_t* base, uint32_t off, __nv_bfloat16 v) {
  *reinterpret_cast<__nv_bfloat16*>(base + off) = v;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// rows [t0, t0 + 128) of this head's dc columns into the staging buffer, 16 bytes per copy (rows at
// or past r_end are not copied: the tile's reads skip them)
__device__ __forceinline__ void stage_dc(uint8_t* smem, const float* dc, long long t0, long long r_end, int W,
                                         int ccol, int tid) {
#pragma unroll
  for (int u = 0; u < CT * CD / 4 / CT_THREADS; ++u) {
    const int c = u * CT_THREADS + tid, r = c / (CD / 4), q = c % (CD / 4);
    if (t0 + r < r_end) cp_async16(smem_u32(smem + OFF_STG + (r * CD + 4 * q) * 4), dc + (t0 + r) * W + ccol + 4 * q);
  }
  cp_async_commit();
}

// bf16 blocks: fp16 latents, bf16 weights (W_c is copied as it is: bf16 is the operand type)
using Tl = __half;
using Tc = __nv_bfloat16;
__global__ void __launch_bounds__(CT_THREADS, 1)
    chanmix_bwd_tc_kernel(const float* __restrict__ dc, const Tl* __restrict__ lat, const Tc* __restrict__ cq_chan,
                          const Tc* __restrict__ ck_chan, const Tc* __restrict__ cq_seq, const Tc* __restrict__ ck_seq,
                          float* __restrict__ ds, float* __restrict__ dwq, float* __restrict__ dwk, long long T, int S,
                          int nq, int nkv, int K, int rows_per_cta, unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* mma_done = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const bool isq = h < nq;
  const int hh = isq ? h : h - nq;
  const int Lq = nq * CD, W = Lq + nkv * CD, Nlat = Lq + 2 * nkv * CD;
  const int ccol = isq ? hh * CD : Lq + hh * CD;
  const Tc* wsrc = (isq ? cq_chan : ck_chan) + (size_t)hh * CD * CD;
  const Tc* wseq = (isq ? cq_seq : ck_seq) + (size_t)hh * CD * K;

  if (tid == 0) {
    mbar_init(smem_u32(mma_done), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  // W_c[i][j] as the MN-major B operand of ds (n = j contiguous, k = i rows): [2 j-halves][128 i][64];
  // 8 columns of a row per copy land in one 16-byte chunk of the swizzled row
#pragma unroll
  for (int u = 0; u < CD * CD / 8 / CT_THREADS; ++u) {
    const int c = u * CT_THREADS + tid, i = c / (CD / 8), j0 = (c % (CD / 8)) * 8;
    cp_async16(smem_u32(smem + OFF_W + (j0 >> 6) * HALF + sw_off(i, j0 & 63)), wsrc + (size_t)i * CD + j0);
  }
  const long long r_begin = (long long)blockIdx.x * rows_per_cta;
  const long long r_end = r_begin + rows_per_cta < T ? r_begin + rows_per_cta : T;
  stage_dc(smem, dc, r_begin, r_end, W, ccol, tid);  // commits W_c's copies too
  // this thread's column j (and row quarter rq of each tile): its seq taps
  const int j = tid % CD, rq = tid / CD;
  float taps[CT_KMAX];
#pragma unroll
  for (int k = 0; k < CT_KMAX; ++k) taps[k] = k < K ? ld_f(wseq + (size_t)j * K + k) : 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const uint32_t idesc_ds = idesc_f32acc(CT, CD, 0, 1, kFmtBF16);  // dc K-major, W_c MN-major
  const uint32_t idesc_dw = idesc_f32acc(CD, CD, 1, 1, kFmtBF16);  // dc and s both read MN-major
  const uint32_t kmaj_hi = desc_hi(smem_desc_sw128(smem_u32(smem), 16, 1024));
  const uint32_t mn_hi = desc_hi(smem_desc_sw128(smem_u32(smem), HALF, 1024));
  const uint32_t dc_lo = desc_lo(smem_desc_sw128(smem_u32(smem + OFF_DC), 16, 1024));
  const uint32_t dcmn_lo = desc_lo(smem_desc_sw128(smem_u32(smem + OFF_DC), HALF, 1024));
  const uint32_t w_lo = desc_lo(smem_desc_sw128(smem_u32(smem + OFF_W), HALF, 1024));
  const uint32_t s_lo = desc_lo(smem_desc_sw128(smem_u32(smem + OFF_S), HALF, 1024));

  bool ok = true;
  uint32_t phase = 0;
  int ntile = 0;
  for (long long t0 = r_begin; t0 < r_end; t0 += CT, ++ntile) {
    // this tile's dc (and, for the first, W_c) in shared memory, from every thread's copies
    cp_async_wait_all();
    __syncthreads();
    // ---- operands of this tile: column j of dc and of s for rows t0 .. t0 + 127
    {
      // win[k] = latent of row t - (K-1) + k, k < K-1 (zero before row 0; taps that reach before a
      // sequence start are skipped below)
      const long long tq = t0 + rq * CT_RROWS;  // this thread's first row
      float win[CT_KMAX];
#pragma unroll
      for (int k = 0; k < CT_KMAX; ++k) {
        const long long row = tq - (K - 1) + k;
        win[k] = (k < K - 1 && row >= 0 && row < T) ? ld_f(lat + row * Nlat + ccol + j) : 0.f;
      }
      int ts = (int)(tq % S);
      const int jh = j >> 6;
#pragma unroll 1
      for (int r0 = rq * CT_RROWS; r0 < (rq + 1) * CT_RROWS; r0 += 8) {
        float dv[8], lv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // independent loads first
          const long long row = t0 + r0 + u;
          const bool in = row < r_end;
          dv[u] = in ? reinterpret_cast<const float*>(smem + OFF_STG)[(r0 + u) * CD + j] : 0.f;
          lv[u] = in ? ld_f(lat + row * Nlat + ccol + j) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float cur = lv[u];
          float sv = 0.f;
#pragma unroll
          for (int k = 0; k < CT_KMAX; ++k)
            if (k < K && ts - (K - 1) + k >= 0) sv = fmaf(taps[k], k == K - 1 ? cur : win[k], sv);
#pragma unroll
          for (int k = 0; k < CT_KMAX - 1; ++k) win[k] = (k < K - 2) ? win[k + 1] : (k == K - 2 ? cur : win[k]);
          const __nv_bfloat16 dh = __float2bfloat16_rn(dv[u]), dl = __float2bfloat16_rn(dv[u] - __bfloat162float(dh));
          const __nv_bfloat16 sh = __float2bfloat16_rn(sv), sl = __float2bfloat16_rn(sv - __bfloat162float(sh));
          const uint32_t o = sw_off(r0 + u, j & 63);
          st_bf16(smem + OFF_DC + jh * HALF, o, dh);
          st_bf16(smem + OFF_DC + (2 + jh) * HALF, o, dl);
          st_bf16(smem + OFF_S + jh * HALF, o, sh);
          st_bf16(smem + OFF_S + (2 + jh) * HALF, o, sl);
          if (++ts == S) ts = 0;
        }
      }
    }
    fence_async_smem();  // the generic-proxy stores above (and W_c's copies) are read by the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // the staging buffer has been read: the next tile's dc comes in while this tile's MMAs run
    if (t0 + CT < r_end) stage_dc(smem, dc, t0 + CT, r_end, W, ccol, tid);
    if (warp == 0) {
      // ds = [dc_hi | dc_lo] [W_c; W_c]: 16 K steps; dc K-major (4 chunks of 64), W_c rows i by 16
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        const uint32_t a = dc_lo + (uint32_t)((((kk >> 2) * HALF) + (kk & 3) * 32) >> 4);
        const uint32_t b = w_lo + (uint32_t)(((kk & 7) * 16 * 128) >> 4);
        if (elect_one_sync()) umma_ss_lohi(tmem, a, kmaj_hi, b, mn_hi, idesc_ds, kk > 0);
      }
      // dW_c += dc_hi s_hi^T + dc_hi s_lo^T + dc_lo s_hi^T: m = i, n = j, k = t (16 rows a step)
#pragma unroll
      for (int seg = 0; seg < 3; ++seg) {
        const uint32_t abase = dcmn_lo + (seg == 2 ? (2 * HALF) >> 4 : 0);
        const uint32_t bbase = s_lo + (seg == 1 ? (2 * HALF) >> 4 : 0);
#pragma unroll
        for (int kk = 0; kk < CT / 16; ++kk) {
          const uint32_t step = (uint32_t)((kk * 16 * 128) >> 4);
          if (elect_one_sync())
            umma_ss_lohi(tmem + CD, abase + step, mn_hi, bbase + step, mn_hi, idesc_dw, ntile > 0 || seg > 0 || kk > 0);
        }
      }
      if (elect_one_sync()) umma_commit(smem_u32(mma_done));
      __syncwarp();
    }
    // every thread leaves the tile loop together if the wait gave up
    const bool waited = mbar_wait_bounded(smem_u32(mma_done), phase, err, nullptr, wait_site(kSiteChanmix, 1, 1));
    if (!__syncthreads_and(waited)) {
      ok = false;
      break;
    }
    phase ^= 1;
    tc_fence_after();
    // ds rows: TMEM lane = row of the tile (warp w reads lanes 32 (w % 4) .., columns 32 (w / 4) ..)
    {
      const int quad = warp & 3;
      const long long row = t0 + quad * 32 + lane;
      const uint32_t base = tmem + ((uint32_t)(quad * 32) << 16);
      {
        const int c = warp >> 2;
        uint32_t v[32];
        tmem_ld_32x32b_x32(base + 32 * c, v);
        tmem_ld_wait();
        if (row < r_end) {
          float* out = ds + row * W + ccol + 32 * c;
#pragma unroll
          for (int m = 0; m < 8; ++m)
            *reinterpret_cast<float4*>(out + 4 * m) =
                make_float4(u2f(v[4 * m]), u2f(v[4 * m + 1]), u2f(v[4 * m + 2]), u2f(v[4 * m + 3]));
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // the shared-memory operands may be overwritten by the next tile
    tc_fence_after();
  }
  // dW_c: TMEM lane = i, columns 128 + j; added to the fp32 sum
  if (ok && ntile > 0) {
    float* dw = (isq ? dwq : dwk) + (size_t)hh * CD * CD;
    const int quad = warp & 3;
    const int i = quad * 32 + lane;
    const uint32_t base = tmem + ((uint32_t)(quad * 32) << 16) + CD;
    {
      const int c = warp >> 2;
      uint32_t v[32];
      tmem_ld_32x32b_x32(base + 32 * c, v);
      tmem_ld_wait();
      float* rowp = dw + (size_t)i * CD + 32 * c;
#pragma unroll
      for (int m = 0; m < 8; ++m)
        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(rowp + 4 * m), "f"(u2f(v[4 * m])),
                     "f"(u2f(v[4 * m + 1])), "f"(u2f(v[4 * m + 2])), "f"(u2f(v[4 * m + 3]))
                     : "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace

bool chanmix_bwd_tc_supported(const BlockDims& dm) {
  return dm.d == CD && dm.K >= 1 && dm.K <= CT_KMAX && dm.io == DType::BF16 && dm.lat == DType::F16;
}

cudaError_t launch_chanmix_bwd_tc(const BlockDims& dm, const float* dc, const void* lat, const void* cq_chan,
                                  const void* ck_chan, const void* cq_seq, const void* ck_seq, float* ds, float* dwq,
                                  float* dwk, unsigned* err, cudaStream_t stream) {
  if (!chanmix_bwd_tc_supported(dm)) return cudaErrorInvalidValue;
  // W_c and dc arrive by 16-byte copies
  if (((reinterpret_cast<uintptr_t>(cq_chan) | reinterpret_cast<uintptr_t>(ck_chan) |
        reinterpret_cast<uintptr_t>(dc)) & 15) != 0)
    return cudaErrorInvalidValue;
  const int heads = dm.nq + dm.nkv;
  // row blocks: about two CTAs per SM over all heads, whole tiles
  long long tiles = (dm.T + CT - 1) / CT;
  long long per = (tiles * heads + 2LL * num_sms() - 1) / (2LL * num_sms());
  if (per < 1) per = 1;
  const int rows = (int)(per * CT);
  const dim3 grid((unsigned)((dm.T + rows - 1) / rows), heads);
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(chanmix_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)CT_SMEM)) !=
      cudaSuccess)
    return e;
  chanmix_bwd_tc_kernel<<<grid, CT_THREADS, CT_SMEM, stream>>>(
      dc, static_cast<const __half*>(lat), static_cast<const __nv_bfloat16*>(cq_chan),
      static_cast<const __nv_bfloat16*>(ck_chan), static_cast<const __nv_bfloat16*>(cq_seq),
      static_cast<const __nv_bfloat16*>(ck_seq), ds, dwq, dwk, dm.T, dm.S, dm.nq, dm.nkv, dm.K, rows, err);
  return cudaGetLastError();
}

}  // namespace cca
