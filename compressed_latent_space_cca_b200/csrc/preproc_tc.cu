// Latent preprocessing of one CCA / CCGQA block for bf16 blocks with
// head_dim 128: the fast path of steps a2-a8 (seq conv, channel conv,
// QK-mean before/after, RoPE, value shift, KV-cache write) in one pass.
//
// "Compressed Convolutional Attention" (gist.science/es/paper/2510.04476),
// section 2.B items 1-3 and section 3 item 2; the exact forms follow the
// readings listed in the project notes (depthwise causal seq conv with tap
// K-1 on the current token, per-head dense channel mix, both QK-mean terms
// added to the conv outputs, rotate-half RoPE, upper half of the V latent
// shifted by one token).
//
// One CTA = 32 tokens of one sequence x one KV group (its G query heads and
// its K/V head). Per head: the fp16 latents of the 32 tokens plus a K-1
// token halo are staged in shared memory, the causal seq conv runs on CUDA
// cores in fp32 and writes an fp16 tile, and the 32x128x128 channel mix runs
// on the tensor cores (mma.sync m16n8k16, fp16 x fp16 -> fp32) against the
// head's weights, converted from bf16 to fp16 while staged. Each thread owns
// the same accumulator positions for every head, so the cross-head QK-mean
// sums stay in registers, and since its columns come in pairs (c, c+64) RoPE
// is applied in registers too. Output tiles are staged in shared memory and
// written with 16-byte coalesced stores: q (fp16), the bf16 K cache and the
// fp16 attention copy of k; then the value shift copies v (bf16 cache and
// fp16 attention copy).
#include <math.h>

#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

constexpr int D = 128;
constexpr int TT = 32;          // tokens per CTA
constexpr int NT = 256;         // threads
constexpr int KMAX = 8;         // largest seq-conv kernel of this path
constexpr int ROWH = D + 8;     // padded row (halves) of the MMA operand tiles: 272 B, ldmatrix conflict-free
constexpr int ZROWS = TT + KMAX - 1;

struct Theta {
  double v[D / 2];  // base^(-2i/d)
};

struct PreParams {
  const __half* lat;       // [T, Nlat] q~ | k~ | v~
  const __nv_bfloat16 *cq_seq, *cq_chan, *ck_seq, *ck_chan;
  __half* q;               // [T, Lq]
  __nv_bfloat16 *k_cache, *v_cache;  // [T, Lkv]
  __half *k_att, *v_att;   // [T, Lkv]
  const __nv_bfloat16* wo;  // [E, Lq] (converted by a side job)
  __half* wo_lat;
  long long wo_n;
  unsigned* err;
  int S, nq, nkv, K, mode, vshift, use_rope;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_f16_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Stage the latents of one head (rows t0-K+1 .. t0+TT-1, zero outside the
// sequence) into zbuf [ZROWS][D] fp16.
__device__ __forceinline__ void load_latents(const PreParams& p, __half* zbuf, long long rowbase, int t0, int col,
                                             int Nlat) {
  const int rows = TT + p.K - 1;
  for (int e = threadIdx.x; e < rows * (D / 8); e += NT) {
    const int r = e / (D / 8), v = e % (D / 8);
    const int t = t0 - (p.K - 1) + r;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (t >= 0 && t < p.S) val = *reinterpret_cast<const uint4*>(p.lat + (rowbase + t) * Nlat + col + v * 8);
    *reinterpret_cast<uint4*>(zbuf + r * D + v * 8) = val;
  }
}

// Stage one head's channel-mix weights [out i][in j] (bf16) as fp16 rows of ROWH.
__device__ __forceinline__ void load_weights(const __nv_bfloat16* W, __half* wbuf, bool& bad) {
  for (int e = threadIdx.x; e < D * (D / 8); e += NT) {
    const int r = e / (D / 8), v = e % (D / 8);
    const uint4 raw = *reinterpret_cast<const uint4*>(W + (long long)r * D + v * 8);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
    uint32_t h[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(b2[k]);
      bad |= f16_overflow(f.x) || f16_overflow(f.y);
      h[k] = pack_f16x2(f.x, f.y);
    }
    *reinterpret_cast<uint4*>(wbuf + r * ROWH + v * 8) = make_uint4(h[0], h[1], h[2], h[3]);
  }
}

// Causal depthwise seq conv of the staged head into sbuf [TT][ROWH] fp16.
__device__ __forceinline__ void seq_conv(const PreParams& p, const __half* zbuf, __half* sbuf,
                                         const __nv_bfloat16* wseq) {
  const int cp = threadIdx.x % (D / 2);  // column pair
  float w0[KMAX], w1[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    w0[j] = j < p.K ? __bfloat162float(wseq[(2 * cp) * p.K + j]) : 0.f;
    w1[j] = j < p.K ? __bfloat162float(wseq[(2 * cp + 1) * p.K + j]) : 0.f;
  }
  for (int t = threadIdx.x / (D / 2); t < TT; t += NT / (D / 2)) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < p.K) {
        const float2 z = __half22float2(*reinterpret_cast<const __half2*>(zbuf + (t + j) * D + 2 * cp));
        a0 = fmaf(w0[j], z.x, a0);
        a1 = fmaf(w1[j], z.y, a1);
      }
    }
    *reinterpret_cast<__half2*>(sbuf + t * ROWH + 2 * cp) = __floats2half2_rn(a0, a1);
  }
}

// Channel mix of the warp's 16 rows x 4 n-tiles: acc[nt][0..3] (m16n8 layout).
__device__ __forceinline__ void channel_mix(const __half* sbuf, const __half* wbuf, int rb, const int* ncol,
                                            float (&acc)[4][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  // ldmatrix addresses: A rows rb + (lane % 16), column block (lane / 16) * 8
  const uint32_t a_base = smem_u32(sbuf + (rb + (lane & 15)) * ROWH + (lane >> 4) * 8);
  // B x4 covers two n-tiles: matrix m = lane / 8 -> n offset (m / 2) * 8, k offset (m % 2) * 8
  const int m = lane >> 3, rr = lane & 7;
  const uint32_t b_base0 = smem_u32(wbuf + (ncol[0] + (m >> 1) * 8 + rr) * ROWH + (m & 1) * 8);
  const uint32_t b_base1 = smem_u32(wbuf + (ncol[2] + (m >> 1) * 8 + rr) * ROWH + (m & 1) * 8);
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    uint32_t a0, a1, a2, a3, b0, b1, b2, b3, c0, c1, c2, c3;
    ldsm_x4(a_base + ks * 32, a0, a1, a2, a3);
    ldsm_x4(b_base0 + ks * 32, b0, b1, b2, b3);
    ldsm_x4(b_base1 + ks * 32, c0, c1, c2, c3);
    mma_f16_16816(acc[0], a0, a1, a2, a3, b0, b1);
    mma_f16_16816(acc[1], a0, a1, a2, a3, b2, b3);
    mma_f16_16816(acc[2], a0, a1, a2, a3, c0, c1);
    mma_f16_16816(acc[3], a0, a1, a2, a3, c2, c3);
  }
}

// Coalesced copy of a staged [TT][ROWH] fp16 tile to rows [t0, t0+TT) of dst (row stride ld).
__device__ __forceinline__ void store_tile_f16(const __half* stage, __half* dst, long long rowbase, int t0, int S,
                                               long long ld) {
  for (int e = threadIdx.x; e < TT * (D / 8); e += NT) {
    const int r = e / (D / 8), v = e % (D / 8);
    if (t0 + r < S)
      *reinterpret_cast<uint4*>(dst + (rowbase + t0 + r) * ld + v * 8) =
          *reinterpret_cast<const uint4*>(stage + r * ROWH + v * 8);
  }
}

__global__ void __launch_bounds__(NT, 2) preproc_tc_kernel(const __grid_constant__ PreParams p,
                                                          const __grid_constant__ Theta th) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __half* kbuf = reinterpret_cast<__half*>(smem_raw);  // [ZROWS][D]  k~ latents (kept)
  __half* zbuf = kbuf + ZROWS * D;                      // [ZROWS][D]  q~ latents of the current head
  __half* wbuf = zbuf + ZROWS * D;                      // [D][ROWH]   channel weights (fp16)
  __half* sbuf = wbuf + D * ROWH;                       // [TT][ROWH]  seq-conv output / output staging
  float* kst = reinterpret_cast<float*>(wbuf);          // [TT][D]     final k (fp32), reuses wbuf

  const int G = p.nq / p.nkv;
  const int Lq = p.nq * D, Lkv = p.nkv * D, Nlat = Lq + 2 * Lkv;
  const int t0 = blockIdx.x * TT, g = blockIdx.y, b = blockIdx.z;
  const long long rowbase = (long long)b * p.S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = (warp & 1) * 16;  // warp rows
  const int cg = warp >> 1;        // column group: cols [16cg, 16cg+16) and the same +64
  const int ncol[4] = {cg * 16, cg * 16 + 8, 64 + cg * 16, 64 + cg * 16 + 8};
  const int r0 = rb + (lane >> 2), r1 = r0 + 8;
  const int cq = (lane & 3) * 2;
  const int zr0 = r0 + p.K - 1, zr1 = r1 + p.K - 1;  // current-token rows in the latent tiles
  bool bad = false;

  // RoPE factors of this thread's (row, column < 64) positions: [nt<2][e]
  float rc[2][4], rs[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = ncol[nt] + cq + (e & 1);
      const int pos = t0 + ((e < 2) ? r0 : r1);
      float c = 1.f, s = 0.f;
      if (p.use_rope) {
        const double a = (double)pos * th.v[i];
        // reduce a modulo 2 pi in two steps (2 pi split into a high and a low part)
        const double k = rint(a * 0.15915494309189535);
        double r = fma(-k, 6.283185307179586, a);
        r = fma(-k, 2.4492935982947064e-16, r);
        sincosf((float)r, &s, &c);
      }
      rc[nt][e] = c;
      rs[nt][e] = s;
    }

  auto rope_pair = [&](float x1, float x2, int nt, int e, float& o1, float& o2) {
    o1 = x1 * rc[nt][e] - x2 * rs[nt][e];
    o2 = x2 * rc[nt][e] + x1 * rs[nt][e];
  };

  // ---- the K head of the group: conv + channel mix, result kept in registers
  float ck[4][4];
  load_latents(p, kbuf, rowbase, t0, Lq + g * D, Nlat);
  load_weights(p.ck_chan + (long long)g * D * D, wbuf, bad);
  __syncthreads();
  seq_conv(p, kbuf, sbuf, p.ck_seq + (long long)g * D * p.K);
  __syncthreads();
  channel_mix(sbuf, wbuf, rb, ncol, ck);

  float csum[4][4], mq[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) csum[nt][e] = mq[nt][e] = 0.f;

  // ---- the G query heads
  for (int hh = 0; hh < G; ++hh) {
    const int h = g * G + hh;
    __syncthreads();  // previous users of zbuf / wbuf / sbuf are done
    load_latents(p, zbuf, rowbase, t0, h * D, Nlat);
    load_weights(p.cq_chan + (long long)h * D * D, wbuf, bad);
    __syncthreads();
    seq_conv(p, zbuf, sbuf, p.cq_seq + (long long)h * D * p.K);
    __syncthreads();
    float acc[4][4];
    channel_mix(sbuf, wbuf, rb, ncol, acc);
    __syncthreads();  // sbuf becomes the output stage
    float val[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = ncol[nt] + cq + (e & 1);
        const int zr = (e < 2) ? zr0 : zr1;
        const float zq = __half2float(zbuf[zr * D + col]);
        const float zk = __half2float(kbuf[zr * D + col]);
        float v = acc[nt][e];
        if (p.mode & 1) v += 0.5f * (zq + zk);
        if (p.mode & 2) v += 0.5f * (acc[nt][e] + ck[nt][e]);
        val[nt][e] = v;
        csum[nt][e] += acc[nt][e];
        mq[nt][e] += zq;
      }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float o1 = val[nt][e], o2 = val[nt + 2][e];
        if (p.use_rope) rope_pair(val[nt][e], val[nt + 2][e], nt, e, o1, o2);
        val[nt][e] = o1;
        val[nt + 2][e] = o2;
      }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int col = ncol[nt] + cq;
      *reinterpret_cast<__half2*>(sbuf + r0 * ROWH + col) = __floats2half2_rn(val[nt][0], val[nt][1]);
      *reinterpret_cast<__half2*>(sbuf + r1 * ROWH + col) = __floats2half2_rn(val[nt][2], val[nt][3]);
#pragma unroll
      for (int e = 0; e < 4; ++e) bad |= f16_overflow(val[nt][e]);
    }
    __syncthreads();
    store_tile_f16(sbuf, p.q + (long long)h * D, rowbase, t0, p.S, Lq);
  }

  // ---- k = c_k + means, RoPE; staged in fp32, written as bf16 cache and fp16 copy
  __syncthreads();  // wbuf is free: it becomes the fp32 k stage
  {
    const float invG = 1.f / (float)G;
    float val[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = ncol[nt] + cq + (e & 1);
        const int zr = (e < 2) ? zr0 : zr1;
        const float zk = __half2float(kbuf[zr * D + col]);
        float v = ck[nt][e];
        if (p.mode & 1) v += 0.5f * (mq[nt][e] * invG + zk);
        if (p.mode & 2) v += 0.5f * (csum[nt][e] * invG + ck[nt][e]);
        val[nt][e] = v;
      }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float o1 = val[nt][e], o2 = val[nt + 2][e];
        if (p.use_rope) rope_pair(val[nt][e], val[nt + 2][e], nt, e, o1, o2);
        val[nt][e] = o1;
        val[nt + 2][e] = o2;
      }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int col = ncol[nt] + cq;
      *reinterpret_cast<float2*>(kst + r0 * D + col) = make_float2(val[nt][0], val[nt][1]);
      *reinterpret_cast<float2*>(kst + r1 * D + col) = make_float2(val[nt][2], val[nt][3]);
#pragma unroll
      for (int e = 0; e < 4; ++e) bad |= f16_overflow(val[nt][e]);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < TT * (D / 8); e += NT) {
    const int r = e / (D / 8), v = e % (D / 8);
    if (t0 + r >= p.S) continue;
    const float* src = kst + r * D + v * 8;
    uint32_t hb[4], hh[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      hb[k] = pack_bf16x2(src[2 * k], src[2 * k + 1]);
      hh[k] = pack_f16x2(src[2 * k], src[2 * k + 1]);
    }
    const long long off = (rowbase + t0 + r) * Lkv + (long long)g * D + v * 8;
    *reinterpret_cast<uint4*>(p.k_cache + off) = make_uint4(hb[0], hb[1], hb[2], hb[3]);
    *reinterpret_cast<uint4*>(p.k_att + off) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
  }

  // ---- value shift: channels [Lkv/2, Lkv) from the previous token (8-channel vectors never straddle)
  for (int e = threadIdx.x; e < TT * (D / 8); e += NT) {
    const int r = e / (D / 8), v = e % (D / 8);
    const int t = t0 + r;
    if (t >= p.S) continue;
    const int gc = g * D + v * 8;
    const int src = (p.vshift && gc >= Lkv / 2) ? t - 1 : t;
    uint4 hv = make_uint4(0, 0, 0, 0);
    if (src >= 0) hv = *reinterpret_cast<const uint4*>(p.lat + (rowbase + src) * Nlat + Lq + Lkv + gc);
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

  // ---- side job: this CTA's slice of W_o as fp16 (8-element vectors)
  {
    const long long nvec = p.wo_n / 8;
    const long long nct = (long long)gridDim.x * gridDim.y * gridDim.z;
    const long long cid = ((long long)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    const long long chunk = (nvec + nct - 1) / nct;
    const long long lo = cid * chunk, hi = lo + chunk < nvec ? lo + chunk : nvec;
    for (long long e = lo + threadIdx.x; e < hi; e += NT) {
      const uint4 raw = *reinterpret_cast<const uint4*>(p.wo + e * 8);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
      uint32_t h[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(b2[k]);
        bad |= f16_overflow(f.x) || f16_overflow(f.y);
        h[k] = pack_f16x2(f.x, f.y);
      }
      *reinterpret_cast<uint4*>(p.wo_lat + e * 8) = make_uint4(h[0], h[1], h[2], h[3]);
    }
  }
  report_range(bad, p.err);
}

constexpr size_t SMEM_BYTES = sizeof(__half) * (2 * ZROWS * D + D * ROWH + TT * ROWH);

}  // namespace

bool preproc_tc_supported(const BlockDims& dm) {
  return dm.io == DType::BF16 && dm.lat == DType::F16 && dm.d == D && dm.K >= 1 && dm.K <= KMAX &&
         ((long long)dm.E * dm.Lq) % 8 == 0;
}

cudaError_t launch_preproc_tc(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream) {
  if (!preproc_tc_supported(dm)) return cudaErrorInvalidValue;
  PreParams q;
  q.lat = static_cast<const __half*>(p.qkv_lat);
  q.cq_seq = static_cast<const __nv_bfloat16*>(p.cq_seq);
  q.cq_chan = static_cast<const __nv_bfloat16*>(p.cq_chan);
  q.ck_seq = static_cast<const __nv_bfloat16*>(p.ck_seq);
  q.ck_chan = static_cast<const __nv_bfloat16*>(p.ck_chan);
  q.q = static_cast<__half*>(p.q);
  q.k_cache = static_cast<__nv_bfloat16*>(p.k_cache);
  q.v_cache = static_cast<__nv_bfloat16*>(p.v_cache);
  q.k_att = static_cast<__half*>(p.k_att);
  q.v_att = static_cast<__half*>(p.v_att);
  q.wo = static_cast<const __nv_bfloat16*>(p.Wo);
  q.wo_lat = static_cast<__half*>(p.wo_lat);
  q.wo_n = (long long)dm.E * dm.Lq;
  q.err = p.dev_err;
  q.S = dm.S;
  q.nq = dm.nq;
  q.nkv = dm.nkv;
  q.K = dm.K;
  q.mode = dm.qk_mean_mode;
  q.vshift = dm.value_shift;
  q.use_rope = dm.use_rope;
  Theta th;
  for (int i = 0; i < D / 2; ++i) th.v[i] = pow((double)dm.rope_base, -2.0 * (double)i / (double)D);
  cudaError_t e = cudaFuncSetAttribute(preproc_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((dm.S + TT - 1) / TT, dm.nkv, dm.B);
  preproc_tc_kernel<<<grid, NT, SMEM_BYTES, stream>>>(q, th);
  return cudaGetLastError();
}

}  // namespace cca
