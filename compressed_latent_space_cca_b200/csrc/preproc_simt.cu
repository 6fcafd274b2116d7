// Latent preprocessing of one CCA / CCGQA block, general SIMT version
// (any even head_dim <= 128; fp32 blocks, or bf16 blocks with fp16
// intermediates; fp32 arithmetic).
//
// "Compressed Convolutional Attention" (gist.science/es/paper/2510.04476),
// section 2.B: on the compressed q~ and k~ a causal convolution along the
// sequence, then a convolution across the channels of each head; the mean of
// q and k taken before and after the convolutions is added; the value shift
// gives half the value channels the previous token. Section 3 item 2: RoPE is
// applied directly in the latent.
//
// One CTA handles TT tokens of one sequence for one KV group g: the G query
// heads of the group and its K/V head, because the QK-mean couples exactly
// those heads. The K-1 tokens before the tile are loaded as a halo.
#include <math.h>

#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

constexpr int PP_TT = 8;       // tokens per CTA
constexpr int PP_THREADS = 256;

// Tl: intermediates (latents in, attention q/k/v out); Tc: weights and KV cache.
template <typename Tl, typename Tc>
__global__ void __launch_bounds__(PP_THREADS) preproc_simt_kernel(
    const Tl* __restrict__ qkv, const Tc* __restrict__ cq_seq, const Tc* __restrict__ cq_chan,
    const Tc* __restrict__ ck_seq, const Tc* __restrict__ ck_chan, Tl* __restrict__ qout, Tc* __restrict__ kout,
    Tc* __restrict__ vout, Tl* __restrict__ katt, Tl* __restrict__ vatt, const Tc* __restrict__ wo,
    Tl* __restrict__ wo_lat, long long wo_n, unsigned* __restrict__ err, int S, int nq, int nkv, int d, int K,
    int mode, int vfrom, int use_rope, float rope_base, int* __restrict__ zero_cnt) {
  extern __shared__ float sm[];
  const int G = nq / nkv;
  const int H1 = G + 1;  // G query heads + the K head of the group
  const int R = PP_TT + K - 1;
  const int Lq = nq * d, Lkv = nkv * d, Nlat = Lq + 2 * Lkv;
  const int half = d / 2;
  float* zin = sm;                       // [H1][R][d]   latents incl. halo
  float* sconv = zin + H1 * R * d;       // [H1][TT][d]  after the seq conv
  float* cconv = sconv + H1 * PP_TT * d; // [H1][TT][d]  after the channel conv
  float* rcos = cconv + H1 * PP_TT * d;  // [TT][d/2]
  float* rsin = rcos + PP_TT * half;     // [TT][d/2]

  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * PP_TT;
  const int g = blockIdx.y, b = blockIdx.z;
  const long long rowbase = (long long)b * S;

  for (int e = tid; e < H1 * R * d; e += PP_THREADS) {
    int hh = e / (R * d), rem = e % (R * d), row = rem / d, i = rem % d;
    int t = t0 - (K - 1) + row;
    int col = (hh < G) ? (g * G + hh) * d + i : Lq + g * d + i;
    zin[e] = (t >= 0 && t < S) ? ld_f(qkv + (rowbase + t) * Nlat + col) : 0.f;
  }
  if (use_rope) {
    const double two_pi = 6.283185307179586476925286766559;
    for (int e = tid; e < PP_TT * half; e += PP_THREADS) {
      int tt = e / half, i = e % half;
      double theta = pow((double)rope_base, -2.0 * (double)i / (double)d);
      double ang = (double)(t0 + tt) * theta;
      double red = ang - two_pi * rint(ang / two_pi);  // exact enough: |ang| < 2^17
      double sv, cv;
      sincos(red, &sv, &cv);
      rcos[e] = (float)cv;
      rsin[e] = (float)sv;
    }
  }
  __syncthreads();

  // causal depthwise conv along the sequence; tap j reads token t-K+1+j
  for (int e = tid; e < H1 * PP_TT * d; e += PP_THREADS) {
    int hh = e / (PP_TT * d), rem = e % (PP_TT * d), tt = rem / d, i = rem % d;
    const Tc* w = (hh < G) ? cq_seq + (long long)((g * G + hh) * d + i) * K : ck_seq + (long long)(g * d + i) * K;
    const float* z = zin + (hh * R + tt) * d + i;
    float acc = 0.f;
    for (int j = 0; j < K; ++j) acc = fmaf(ld_f(w + j), z[j * d], acc);
    sconv[e] = acc;
  }
  __syncthreads();

  // per-head channel mix: one warp per output channel, lanes split the sum
  {
    const int warp = tid >> 5, lane = tid & 31, nwarps = PP_THREADS / 32;
    for (int row = warp; row < H1 * d; row += nwarps) {
      int hh = row / d, i = row % d;
      const Tc* W = (hh < G) ? cq_chan + ((long long)(g * G + hh) * d + i) * d : ck_chan + ((long long)g * d + i) * d;
      float wv[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        int j = lane + 32 * m;
        wv[m] = (j < d) ? ld_f(W + j) : 0.f;
      }
      for (int tt = 0; tt < PP_TT; ++tt) {
        const float* s = sconv + (hh * PP_TT + tt) * d;
        float part = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          int j = lane + 32 * m;
          if (j < d) part = fmaf(wv[m], s[j], part);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        if (lane == 0) cconv[(hh * PP_TT + tt) * d + i] = part;
      }
    }
  }
  __syncthreads();

  // QK-mean (before / after the convs), RoPE, store q and the K cache
  const float invG = 1.f / (float)G;
  auto combined = [&](int hh, int tt, int i) -> float {
    const float c = cconv[(hh * PP_TT + tt) * d + i];
    const float zc = zin[(hh * R + tt + K - 1) * d + i];
    float r = c;
    if (hh < G) {
      if (mode & 1) r += 0.5f * (zc + zin[(G * R + tt + K - 1) * d + i]);
      if (mode & 2) r += 0.5f * (c + cconv[(G * PP_TT + tt) * d + i]);
    } else {
      if (mode & 1) {
        float mq = 0.f;
        for (int h2 = 0; h2 < G; ++h2) mq += zin[(h2 * R + tt + K - 1) * d + i];
        r += 0.5f * (mq * invG + zc);
      }
      if (mode & 2) {
        float mc = 0.f;
        for (int h2 = 0; h2 < G; ++h2) mc += cconv[(h2 * PP_TT + tt) * d + i];
        r += 0.5f * (mc * invG + c);
      }
    }
    return r;
  };
  bool bad = false;
  for (int e0 = 0; e0 < H1 * PP_TT * half; e0 += PP_THREADS) {
    const int e = e0 + tid;
    int hh = e / (PP_TT * half), rem = e % (PP_TT * half), tt = rem / half, i = rem % half;
    int t = t0 + tt;
    if (e < H1 * PP_TT * half && t < S) {
      float x1 = combined(hh, tt, i), x2 = combined(hh, tt, i + half);
      float o1 = x1, o2 = x2;
      if (use_rope) {
        float c = rcos[tt * half + i], s = rsin[tt * half + i];
        o1 = x1 * c - x2 * s;
        o2 = x2 * c + x1 * s;
      }
      if (hh < G) {
        Tl* dst = qout + (rowbase + t) * Lq + (long long)(g * G + hh) * d;
        st_f(dst + i, o1);
        st_f(dst + i + half, o2);
      } else {
        Tc* dst = kout + (rowbase + t) * Lkv + (long long)g * d;
        st_f(dst + i, o1);
        st_f(dst + i + half, o2);
        if (katt != nullptr) {
          Tl* da = katt + (rowbase + t) * Lkv + (long long)g * d;
          st_f(da + i, o1);
          st_f(da + i + half, o2);
        }
      }
      if (sizeof(Tl) == 2) bad |= f16_overflow(o1) || f16_overflow(o2);
    }
  }

  // value shift: channels [vfrom, Lkv) come from the previous token (vfrom = Lkv: no shift)
  for (int e = tid; e < PP_TT * d; e += PP_THREADS) {
    int tt = e / d, i = e % d;
    int t = t0 + tt;
    if (t >= S) continue;
    int gc = g * d + i;
    int src = gc >= vfrom ? t - 1 : t;
    const float val = (src >= 0) ? ld_f(qkv + (rowbase + src) * Nlat + Lq + Lkv + gc) : 0.f;
    st_f(vout + (rowbase + t) * Lkv + gc, val);
    if (vatt != nullptr) st_f(vatt + (rowbase + t) * Lkv + gc, val);
  }

  // side job: this CTA's slice of the W_o copy in the intermediate type
  if (wo_lat != nullptr) {
    const long long nct = (long long)gridDim.x * gridDim.y * gridDim.z;
    const long long cid = ((long long)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    const long long chunk = (wo_n + nct - 1) / nct;
    const long long lo = cid * chunk, hi = lo + chunk < wo_n ? lo + chunk : wo_n;
    for (long long e = lo + tid; e < hi; e += PP_THREADS) {
      const float w = ld_f(wo + e);
      st_f(wo_lat + e, w);
      bad |= f16_overflow(w);
    }
  }
  // side job: clear the attention's split-pair counters for the launch that follows
  if (zero_cnt != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
    for (int i = tid; i < kAttnSplitCounters; i += PP_THREADS) zero_cnt[i] = 0;
  report_range(bad, err);
}

// Conv state per sequence: the last K-1 rows of q~ and of k~ and the last row
// of v~, zero rows before the sequence start.
template <typename Tl, typename Tc>
__global__ void conv_state_kernel(const Tl* __restrict__ qkv, Tc* __restrict__ state, int S, int Lq, int Lkv,
                                  int K) {
  const int b = blockIdx.x;
  const int Nlat = Lq + 2 * Lkv;
  const long long per = (long long)(K - 1) * (Lq + Lkv) + Lkv;
  Tc* dst = state + b * per;
  const long long rowbase = (long long)b * S;
  for (long long e = threadIdx.x; e < per; e += blockDim.x) {
    int t, col;
    if (e < (long long)(K - 1) * Lq) {
      t = S - (K - 1) + (int)(e / Lq);
      col = (int)(e % Lq);
    } else if (e < (long long)(K - 1) * (Lq + Lkv)) {
      long long e2 = e - (long long)(K - 1) * Lq;
      t = S - (K - 1) + (int)(e2 / Lkv);
      col = Lq + (int)(e2 % Lkv);
    } else {
      t = S - 1;
      col = Lq + Lkv + (int)(e - (long long)(K - 1) * (Lq + Lkv));
    }
    st_f(dst + e, t >= 0 ? ld_f(qkv + (rowbase + t) * Nlat + col) : 0.f);
  }
}

}  // namespace

namespace {
template <typename Tl, typename Tc>
cudaError_t preproc_typed(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream) {
  const int H1 = dm.G + 1, R = PP_TT + dm.K - 1;
  size_t smem = sizeof(float) * ((size_t)H1 * R * dm.d + 2 * (size_t)H1 * PP_TT * dm.d + (size_t)PP_TT * dm.d);
  dim3 grid((dm.S + PP_TT - 1) / PP_TT, dm.nkv, dm.B);
  auto kern = preproc_simt_kernel<Tl, Tc>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const bool sep = dm.lat != dm.io;  // separate attention K/V and W_o copies
  kern<<<grid, PP_THREADS, smem, stream>>>(
      (const Tl*)p.qkv_lat, (const Tc*)p.cq_seq, (const Tc*)p.cq_chan, (const Tc*)p.ck_seq, (const Tc*)p.ck_chan,
      (Tl*)p.q, (Tc*)p.k_cache, (Tc*)p.v_cache, sep ? (Tl*)p.k_att : nullptr, sep ? (Tl*)p.v_att : nullptr,
      (const Tc*)p.Wo, sep ? (Tl*)p.wo_lat : nullptr, (long long)dm.E * dm.Lq, p.dev_err, dm.S, dm.nq, dm.nkv, dm.d,
      dm.K, dm.qk_mean_mode, dm.value_shift ? dm.vshift_from : dm.Lkv, dm.use_rope, dm.rope_base,
      attention_tc_supported(dm) ? static_cast<int*>(p.sched) : nullptr);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_preproc_simt(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream) {
  if (dm.io == DType::BF16 && dm.lat == DType::F16) return preproc_typed<__half, __nv_bfloat16>(dm, p, stream);
  if (dm.io == DType::F32 && dm.lat == DType::F32) return preproc_typed<float, float>(dm, p, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_conv_state(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream) {
  if (p.conv_state == nullptr) return cudaSuccess;
  if (dm.io == DType::BF16 && dm.lat == DType::F16)
    conv_state_kernel<__half, __nv_bfloat16><<<dm.B, 256, 0, stream>>>(
        (const __half*)p.qkv_lat, (__nv_bfloat16*)p.conv_state, dm.S, dm.Lq, dm.Lkv, dm.K);
  else if (dm.io == DType::F32 && dm.lat == DType::F32)
    conv_state_kernel<float, float><<<dm.B, 256, 0, stream>>>((const float*)p.qkv_lat, (float*)p.conv_state, dm.S,
                                                              dm.Lq, dm.Lkv, dm.K);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace cca
