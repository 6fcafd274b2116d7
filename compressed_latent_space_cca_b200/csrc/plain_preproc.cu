// Preprocessing of a plain attention block (conv_kernel 0): q, k and v come straight from the
// projections, without the convolutions, QK-mean or value shift of a CCA block. This is the
// uncompressed multi-head (C = 1) or grouped-query baseline that "Compressed Convolutional
// Attention" (gist.science/es/paper/2510.04476, section 4) compares CCA against; RoPE is the same
// rotate-half form the CCA block applies in its latent (section 3 item 2).
//
// One CTA = 32 tokens of one sequence. The CTA first tabulates (cos, sin) of position x theta_i
// for its tokens (angles reduced modulo 2 pi in fp64), then walks the token rows: for every q and
// k head the pair (i, i + d/2) is rotated, for every v head each element is copied. Consecutive
// threads take consecutive i, so every global access of a warp is contiguous. Outputs: q (the
// attention input, intermediate type), the KV cache (block type) and, for bf16 blocks, the fp16
// attention copies of k and v. Side jobs as in the other preprocessing kernels: a slice of the
// fp16 copy of W_o and the attention's split-pair counters.
#include <math.h>

#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

constexpr int PT = 32;    // tokens per CTA
constexpr int PNT = 256;  // threads
constexpr int MAXHALF = 64;

struct PlainParams {
  const void* lat;  // [T, Nlat] q~ | k~ | v~ (intermediate type)
  void *q, *k_cache, *v_cache, *k_att, *v_att;
  const void* wo;
  void* wo_lat;
  long long wo_n;
  int* zero_cnt;
  unsigned* err;
  int S, nq, nkv, d, use_rope, sep;
  double theta[MAXHALF];  // base^(-2i/d)
};

// VEC: bf16 blocks with d % 16 == 0 handle 8 consecutive pairs (or 8 v elements) per item with
// 16-byte accesses; otherwise one pair (or one element) per item.
template <typename Tl, typename Tc, bool VEC>
__global__ void __launch_bounds__(PNT) plain_preproc_kernel(const __grid_constant__ PlainParams p) {
  __shared__ float2 rtab[PT][MAXHALF];  // (cos, sin) of (t0 + r) * theta_i
  const int t0 = blockIdx.x * PT, b = blockIdx.y;
  const int half = p.d / 2;
  const int Lq = p.nq * p.d, Lkv = p.nkv * p.d, Nlat = Lq + 2 * Lkv;
  const long long rowbase = (long long)b * p.S;
  const Tl* lat = static_cast<const Tl*>(p.lat);
  if (p.use_rope) {
    for (int e = threadIdx.x; e < PT * half; e += PNT) {
      const int r = e / half, i = e % half;
      const double a = (double)(t0 + r) * p.theta[i];
      // reduce a modulo 2 pi with 2 pi split into a high and a low double
      const double k = rint(a * 0.15915494309189535);
      double x = fma(-k, 6.283185307179586, a);
      x = fma(-k, 2.4492935982947064e-16, x);
      float sn, cs;
      sincosf((float)x, &sn, &cs);
      rtab[r][i] = make_float2(cs, sn);
    }
    __syncthreads();
  }
  float amax = 0.f;  // largest |value| written in the intermediate type
  const int rows = p.S - t0 < PT ? p.S - t0 : PT;
  if constexpr (VEC) {
    const int hv = half / 8;                                    // 8-pair groups per head
    const int nrot = (p.nq + p.nkv) * hv, nrow = nrot + Lkv / 8;  // items per token row
    for (int e = threadIdx.x; e < rows * nrow; e += PNT) {
      const int r = e / nrow, j = e - r * nrow;
      const long long row = rowbase + t0 + r;
      const __half* src = reinterpret_cast<const __half*>(lat) + row * Nlat;
      if (j < nrot) {
        const int head = j / hv, i0 = (j - head * hv) * 8;
        const bool isq = head < p.nq;
        const int col = isq ? head * p.d + i0 : Lq + (head - p.nq) * p.d + i0;
        const uint4 a = *reinterpret_cast<const uint4*>(src + col), c = *reinterpret_cast<const uint4*>(src + col + half);
        const __half2* a2 = reinterpret_cast<const __half2*>(&a);
        const __half2* c2 = reinterpret_cast<const __half2*>(&c);
        float y1[8], y2[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 x1 = __half22float2(a2[u]), x2 = __half22float2(c2[u]);
          y1[2 * u] = x1.x;
          y1[2 * u + 1] = x1.y;
          y2[2 * u] = x2.x;
          y2[2 * u + 1] = x2.y;
        }
        if (p.use_rope) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float2 cs = rtab[r][i0 + u];
            const float v1 = y1[u] * cs.x - y2[u] * cs.y, v2 = y2[u] * cs.x + y1[u] * cs.y;
            y1[u] = v1;
            y2[u] = v2;
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) amax = fmaxf(amax, fmaxf(fabsf(y1[u]), fabsf(y2[u])));
        const uint4 h1 = make_uint4(pack_f16x2(y1[0], y1[1]), pack_f16x2(y1[2], y1[3]), pack_f16x2(y1[4], y1[5]),
                                    pack_f16x2(y1[6], y1[7]));
        const uint4 h2 = make_uint4(pack_f16x2(y2[0], y2[1]), pack_f16x2(y2[2], y2[3]), pack_f16x2(y2[4], y2[5]),
                                    pack_f16x2(y2[6], y2[7]));
        if (isq) {
          __half* dq = static_cast<__half*>(p.q) + row * Lq + head * p.d + i0;
          *reinterpret_cast<uint4*>(dq) = h1;
          *reinterpret_cast<uint4*>(dq + half) = h2;
        } else {
          const long long off = row * Lkv + (head - p.nq) * p.d + i0;
          __nv_bfloat16* kc = static_cast<__nv_bfloat16*>(p.k_cache) + off;
          *reinterpret_cast<uint4*>(kc) = make_uint4(pack_bf16x2(y1[0], y1[1]), pack_bf16x2(y1[2], y1[3]),
                                                     pack_bf16x2(y1[4], y1[5]), pack_bf16x2(y1[6], y1[7]));
          *reinterpret_cast<uint4*>(kc + half) = make_uint4(pack_bf16x2(y2[0], y2[1]), pack_bf16x2(y2[2], y2[3]),
                                                            pack_bf16x2(y2[4], y2[5]), pack_bf16x2(y2[6], y2[7]));
          __half* ka = static_cast<__half*>(p.k_att) + off;
          *reinterpret_cast<uint4*>(ka) = h1;
          *reinterpret_cast<uint4*>(ka + half) = h2;
        }
      } else {  // copy 8 v elements
        const int c0 = (j - nrot) * 8;
        const uint4 v = *reinterpret_cast<const uint4*>(src + Lq + Lkv + c0);
        const __half2* v2 = reinterpret_cast<const __half2*>(&v);
        uint32_t b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 f = __half22float2(v2[u]);
          b[u] = pack_bf16x2(f.x, f.y);
        }
        const long long off = row * Lkv + c0;
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.v_cache) + off) = make_uint4(b[0], b[1], b[2], b[3]);
        *reinterpret_cast<uint4*>(static_cast<__half*>(p.v_att) + off) = v;
      }
    }
  }
  const int nrot = (p.nq + p.nkv) * half, nrow = nrot + Lkv;  // items per token row (scalar path)
  for (int e = VEC ? rows * nrow : threadIdx.x; e < rows * nrow; e += PNT) {
    const int r = e / nrow, j = e - r * nrow;
    const long long row = rowbase + t0 + r;
    const Tl* src = lat + row * Nlat;
    if (j < nrot) {  // rotate (i, i + d/2) of a q head, then of a k head
      const int head = j / half, i = j % half;
      const bool isq = head < p.nq;
      const int col = isq ? head * p.d + i : Lq + (head - p.nq) * p.d + i;
      float x1 = ld_f(src + col), x2 = ld_f(src + col + half);
      if (p.use_rope) {
        const float2 cs = rtab[r][i];
        const float y1 = x1 * cs.x - x2 * cs.y, y2 = x2 * cs.x + x1 * cs.y;
        x1 = y1;
        x2 = y2;
      }
      if (isq) {
        Tl* dq = static_cast<Tl*>(p.q) + row * Lq + head * p.d + i;
        st_f(dq, x1);
        st_f(dq + half, x2);
        amax = fmaxf(amax, fmaxf(fabsf(x1), fabsf(x2)));
      } else {
        const long long off = row * Lkv + (head - p.nq) * p.d + i;
        st_f(static_cast<Tc*>(p.k_cache) + off, x1);
        st_f(static_cast<Tc*>(p.k_cache) + off + half, x2);
        if (p.sep) {
          st_f(static_cast<Tl*>(p.k_att) + off, x1);
          st_f(static_cast<Tl*>(p.k_att) + off + half, x2);
          amax = fmaxf(amax, fmaxf(fabsf(x1), fabsf(x2)));
        }
      }
    } else {  // copy v
      const int c = j - nrot;
      const float v = ld_f(src + Lq + Lkv + c);
      const long long off = row * Lkv + c;
      st_f(static_cast<Tc*>(p.v_cache) + off, v);
      if (p.sep) st_f(static_cast<Tl*>(p.v_att) + off, v);
    }
  }
  bool bad = false;
  // side job: this CTA's slice of the W_o copy in the intermediate type
  if (p.wo_lat != nullptr) {
    const long long nct = (long long)gridDim.x * gridDim.y;
    const long long cid = (long long)blockIdx.y * gridDim.x + blockIdx.x;
    const long long chunk = (p.wo_n + nct - 1) / nct;
    const long long lo = cid * chunk, hi = lo + chunk < p.wo_n ? lo + chunk : p.wo_n;
    for (long long e = lo + threadIdx.x; e < hi; e += PNT) {
      const float w = ld_f(static_cast<const Tc*>(p.wo) + e);
      st_f(static_cast<Tl*>(p.wo_lat) + e, w);
      bad |= f16_overflow(w);
    }
  }
  // side job: clear the attention's split-pair counters for the launch that follows
  if (p.zero_cnt != nullptr && blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = threadIdx.x; i < kAttnSplitCounters; i += PNT) p.zero_cnt[i] = 0;
  if (sizeof(Tl) == 2) bad |= amax > 65504.0f;  // fp16 intermediates, infinities included
  report_range(bad, p.err);
}

}  // namespace

cudaError_t launch_plain_preproc(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream) {
  if (dm.K != 0 || dm.d / 2 > MAXHALF) return cudaErrorInvalidValue;
  PlainParams q{};
  q.lat = p.qkv_lat;
  q.q = p.q;
  q.k_cache = p.k_cache;
  q.v_cache = p.v_cache;
  q.k_att = p.k_att;
  q.v_att = p.v_att;
  q.sep = dm.lat != dm.io;
  q.wo = p.Wo;
  q.wo_lat = q.sep ? p.wo_lat : nullptr;
  q.wo_n = (long long)dm.E * dm.Lq;
  q.zero_cnt = attention_tc_supported(dm) ? static_cast<int*>(p.sched) : nullptr;
  q.err = p.dev_err;
  q.S = dm.S;
  q.nq = dm.nq;
  q.nkv = dm.nkv;
  q.d = dm.d;
  q.use_rope = dm.use_rope;
  for (int i = 0; i < dm.d / 2; ++i) q.theta[i] = pow((double)dm.rope_base, -2.0 * (double)i / (double)dm.d);
  dim3 grid((dm.S + PT - 1) / PT, dm.B);
  if (dm.io == DType::BF16 && dm.lat == DType::F16) {
    if (dm.d % 16 == 0)
      plain_preproc_kernel<__half, __nv_bfloat16, true><<<grid, PNT, 0, stream>>>(q);
    else
      plain_preproc_kernel<__half, __nv_bfloat16, false><<<grid, PNT, 0, stream>>>(q);
  } else if (dm.io == DType::F32 && dm.lat == DType::F32) {
    plain_preproc_kernel<float, float, false><<<grid, PNT, 0, stream>>>(q);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace cca
