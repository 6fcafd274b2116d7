// The backward pass of one CCA / CCGQA block: given dL/dy, the gradients of x and of every weight
// ("Compressed Convolutional Attention", gist.science/es/paper/2510.04476, section 4 reports the
// backward of CCGQA; its form is the chain rule through the forward of section 2 in reverse).
//
// The forward's activations are recomputed by the forward kernels into the backward's workspace;
// then, in fp32:
//   dO = dy W_o;  dW_o = dy^T O                                  (strided GEMMs)
//   per (row, head): LSE of the softmax and delta = rowsum(dO o O)
//   attention backward (FlashAttention-2 form): a CTA per 64-key block of one KV group walks the
//     query blocks at or after it for each query head of the group, recomputes P from q, k and the
//     LSE, accumulates dV and dK in registers and adds dQ atomically
//   per token: RoPE turned back, the QK-mean terms' transpose (which feeds dc and the latents
//     directly), the value shift's transpose
//   channel mix: ds = W_c^T dc, dW_c = sum_t dc^T s (s recomputed from the latents)
//   seq conv: dz[t] = sum_j w_j ds[t + K-1-j], dw_j = sum_t ds[t] z[t-K+1+j]
//   down-projection: dx = dlat [W_q; W_k; W_v], dW = dlat^T x       (strided GEMMs)
// Every product here runs on the CUDA cores in fp32 (a first form of this pass: correct, not fast).
#include <math.h>

#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

// ------------------------------------------------------------------ strided GEMM --
// C[z][m][n] (+)= sum_k A[z][m*sam + k*sak] * B[z][n*sbn + k*sbk] in fp32, for a batch of z problems
// whose operands start zsa, zsb and zsc elements apart. 64 x 64 tiles, 16-deep K steps, 256 threads
// with 4 x 4 outputs each. With ksplit > 1 the K range is cut into ksplit slices (grid z = batch x
// ksplit) whose partial sums are added atomically into C.
constexpr int SG_M = 64, SG_N = 64, SG_K = 16;

template <typename TA, typename TB>
__global__ void __launch_bounds__(256) gemm_strided_kernel(const TA* __restrict__ A, long long sam, long long sak,
                                                           long long zsa, const TB* __restrict__ B, long long sbn,
                                                           long long sbk, long long zsb, float* __restrict__ C,
                                                           long long ldc, long long zsc, int M, int N, long long K,
                                                           int accumulate, int ksplit) {
  __shared__ float As[SG_K][SG_M + 4];
  __shared__ float Bs[SG_K][SG_N + 4];
  const int tid = threadIdx.x;
  const long long z = blockIdx.z / ksplit;
  const int slice = blockIdx.z % ksplit;
  A += z * zsa;
  B += z * zsb;
  C += z * zsc;
  const int m0 = blockIdx.y * SG_M, n0 = blockIdx.x * SG_N;
  const int tr = tid / 16, tc = tid % 16;
  const long long kchunk = ((K + ksplit - 1) / ksplit + SG_K - 1) / SG_K * SG_K;
  const long long kbeg = slice * kchunk, kend = kbeg + kchunk < K ? kbeg + kchunk : K;
  float acc[4][4] = {};
  for (long long k0 = kbeg; k0 < kend; k0 += SG_K) {
    // each thread loads 4 elements of each tile; the fastest-moving index follows the operand's
    // unit stride where it has one
    for (int e = tid; e < SG_K * SG_M; e += 256) {
      int kk, mm;
      if (sam == 1) {
        mm = e % SG_M;
        kk = e / SG_M;
      } else {
        kk = e % SG_K;
        mm = e / SG_K;
      }
      const long long k = k0 + kk;
      const int m = m0 + mm;
      As[kk][mm] = (m < M && k < kend) ? ld_f(A + m * sam + k * sak) : 0.f;
    }
    for (int e = tid; e < SG_K * SG_N; e += 256) {
      int kk, nn;
      if (sbn == 1) {
        nn = e % SG_N;
        kk = e / SG_N;
      } else {
        kk = e % SG_K;
        nn = e / SG_K;
      }
      const long long k = k0 + kk;
      const int n = n0 + nn;
      Bs[kk][nn] = (n < N && k < kend) ? ld_f(B + n * sbn + k * sbk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG_K; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][tr * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tc * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + tr * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tc * 4 + j;
      if (n >= N) continue;
      float* c = C + (long long)m * ldc + n;
      if (ksplit > 1) atomicAdd(c, acc[i][j]);
      else *c = accumulate ? *c + acc[i][j] : acc[i][j];
    }
  }
}

struct Mat {
  const void* p;
  DType t;
};

template <typename TA>
cudaError_t gemm_b(Mat a, long long sam, long long sak, long long zsa, Mat b, long long sbn, long long sbk,
                   long long zsb, float* C, long long ldc, long long zsc, int M, int N, long long K, int batch,
                   bool accumulate, int ksplit, cudaStream_t s) {
  const dim3 grid((N + SG_N - 1) / SG_N, (M + SG_M - 1) / SG_M, batch * ksplit);
  const TA* A = static_cast<const TA*>(a.p);
  switch (b.t) {
    case DType::F32:
      gemm_strided_kernel<TA, float><<<grid, 256, 0, s>>>(A, sam, sak, zsa, static_cast<const float*>(b.p), sbn, sbk,
                                                          zsb, C, ldc, zsc, M, N, K, accumulate, ksplit);
      break;
    case DType::BF16:
      gemm_strided_kernel<TA, __nv_bfloat16><<<grid, 256, 0, s>>>(A, sam, sak, zsa,
                                                                  static_cast<const __nv_bfloat16*>(b.p), sbn, sbk,
                                                                  zsb, C, ldc, zsc, M, N, K, accumulate, ksplit);
      break;
    case DType::F16:
      gemm_strided_kernel<TA, __half><<<grid, 256, 0, s>>>(A, sam, sak, zsa, static_cast<const __half*>(b.p), sbn,
                                                           sbk, zsb, C, ldc, zsc, M, N, K, accumulate, ksplit);
      break;
  }
  return cudaGetLastError();
}

// A long K (the token dimension of a weight gradient) with few output tiles is split so that the
// grid covers the SMs about twice; C (a contiguous [batch][M][ldc] block) is cleared first unless
// it accumulates.
cudaError_t gemm(Mat a, long long sam, long long sak, long long zsa, Mat b, long long sbn, long long sbk, long long zsb,
                 float* C, long long ldc, long long zsc, int M, int N, long long K, int batch, bool accumulate,
                 cudaStream_t s) {
  const long long tiles = (long long)((N + SG_N - 1) / SG_N) * ((M + SG_M - 1) / SG_M) * batch;
  const long long want = (2LL * num_sms() + tiles - 1) / tiles;
  long long ksplit = want < K / 512 ? want : K / 512;
  if (ksplit < 1) ksplit = 1;
  if (ksplit > 1 && !accumulate) {
    const long long n = (long long)(batch - 1) * zsc + (long long)(M - 1) * ldc + N;
    const cudaError_t e = cudaMemsetAsync(C, 0, sizeof(float) * n, s);
    if (e != cudaSuccess) return e;
  }
  const int ks = (int)ksplit;
  switch (a.t) {
    case DType::F32: return gemm_b<float>(a, sam, sak, zsa, b, sbn, sbk, zsb, C, ldc, zsc, M, N, K, batch, accumulate, ks, s);
    case DType::BF16:
      return gemm_b<__nv_bfloat16>(a, sam, sak, zsa, b, sbn, sbk, zsb, C, ldc, zsc, M, N, K, batch, accumulate, ks, s);
    case DType::F16:
      return gemm_b<__half>(a, sam, sak, zsa, b, sbn, sbk, zsb, C, ldc, zsc, M, N, K, batch, accumulate, ks, s);
  }
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ row statistics --
// Per (row t, query head h): lse = m + log(l) of the causal softmax of scale * q k^T (base e), and
// delta = sum_i dO[t,h,i] O[t,h,i]. A CTA per (64-row block, head, sequence) walks the key blocks
// at or before it: each thread holds a 4 x 4 patch of the score tile, rows are reduced over the 16
// threads that share them, and every thread keeps the running (m, l) of its 4 rows.
constexpr int RB = 64;

template <typename Tl>
__global__ void __launch_bounds__(256, 2) row_stats_kernel(const Tl* __restrict__ q, const Tl* __restrict__ k,
                                                        const Tl* __restrict__ o, const float* __restrict__ dO,
                                                        float* __restrict__ lse, float* __restrict__ delta, int S,
                                                        int nq, int nkv, int d, float scale) {
  extern __shared__ float rsm[];
  const int DP = d + 1;  // padded rows: the 16 rows a warp reads fall in different banks
  float* qs = rsm;           // [RB][DP]
  float* ks = qs + RB * DP;  // [RB][DP]
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = nq / nkv, g = h / G, Lq = nq * d, Lkv = nkv * d;
  const long long rb = (long long)b * S;
  const int q0 = qb * RB, tid = threadIdx.x;
  const int qr = tid / 16, kc = tid % 16;
  for (int e = tid; e < RB * d; e += 256) {
    const int r = e / d, c = e % d;
    qs[r * DP + c] = q0 + r < S ? ld_f(q + (rb + q0 + r) * Lq + h * d + c) : 0.f;
  }
  float m[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
  }
  for (int k0 = 0; k0 <= q0; k0 += RB) {
    __syncthreads();
    for (int e = tid; e < RB * d; e += 256) {
      const int r = e / d, c = e % d;
      ks[r * DP + c] = k0 + r < S ? ld_f(k + (rb + k0 + r) * Lkv + g * d + c) : 0.f;
    }
    __syncthreads();
    float sacc[4][4] = {};
    for (int c = 0; c < d; ++c) {
      float qa[4], kb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        qa[i] = qs[(qr * 4 + i) * DP + c];
        kb[i] = ks[(kc * 4 + i) * DP + c];
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) sacc[a][bb] = fmaf(qa[a], kb[bb], sacc[a][bb]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int t = q0 + qr * 4 + a;
      float mx = -INFINITY;
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        const int key = k0 + kc * 4 + bb;
        sacc[a][bb] = (key <= t && key < S) ? sacc[a][bb] * scale : -INFINITY;
        mx = fmaxf(mx, sacc[a][bb]);
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float mn = fmaxf(m[a], mx);
      float sum = 0.f;
      if (mn != -INFINITY) {
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) sum += sacc[a][bb] == -INFINITY ? 0.f : expf(sacc[a][bb] - mn);
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      l[a] = (m[a] == -INFINITY ? 0.f : l[a] * expf(m[a] - mn)) + sum;
      m[a] = mn;
    }
  }
  if (kc == 0) {
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int t = q0 + qr * 4 + a;
      if (t < S) lse[(rb + t) * nq + h] = m[a] + logf(l[a]);
    }
  }
  // delta: 4 threads per row, each over a quarter of the columns
  {
    const int r = tid / 4, part = tid % 4;
    float dl = 0.f;
    if (q0 + r < S) {
      const Tl* orow = o + (rb + q0 + r) * Lq + h * d;
      const float* drow = dO + (rb + q0 + r) * Lq + h * d;
      for (int c = part; c < d; c += 4) dl = fmaf(ld_f(orow + c), drow[c], dl);
    }
    dl += __shfl_xor_sync(0xffffffffu, dl, 1);
    dl += __shfl_xor_sync(0xffffffffu, dl, 2);
    if (part == 0 && q0 + r < S) delta[(rb + q0 + r) * nq + h] = dl;
  }
}

// dO in fp16 for the tensor-core attention backward, and delta_t = sum_i dO[t,h,i] O[t,h,i] in the
// [B][nq][stride] layout it reads. A warp per (row, head) of head_dim 128: four columns a lane.
__global__ void __launch_bounds__(256) do_prep_kernel(const float* __restrict__ dO, const __half* __restrict__ o,
                                                      __half* __restrict__ dO16, float* __restrict__ delta, long long T,
                                                      int S, int nq, int stride, __nv_bfloat16* __restrict__ o_planes,
                                                      long long Tp) {
  const long long wid = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= T * nq) return;
  const long long row = wid / nq;
  const int h = (int)(wid % nq);
  const long long off = row * nq * 128 + h * 128 + lane * 4;
  const float4 g = *reinterpret_cast<const float4*>(dO + off);
  const uint2 ov = *reinterpret_cast<const uint2*>(o + off);
  const __half2 o01 = *reinterpret_cast<const __half2*>(&ov.x), o23 = *reinterpret_cast<const __half2*>(&ov.y);
  float dl = g.x * __low2float(o01) + g.y * __high2float(o01) + g.z * __low2float(o23) + g.w * __high2float(o23);
  *reinterpret_cast<uint2*>(dO16 + off) = make_uint2(pack_f16x2(g.x, g.y), pack_f16x2(g.z, g.w));
  if (o_planes != nullptr) {  // O as bf16 hi / lo planes [2][Tp][Lq] (the dW_o GEMM's operand)
    const float of[4] = {__low2float(o01), __high2float(o01), __low2float(o23), __high2float(o23)};
    float hf[4], lf[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat16 hb = __float2bfloat16_rn(of[u]);
      hf[u] = __bfloat162float(hb);
      lf[u] = of[u] - hf[u];
    }
    *reinterpret_cast<uint2*>(o_planes + off) = make_uint2(pack_bf16x2(hf[0], hf[1]), pack_bf16x2(hf[2], hf[3]));
    *reinterpret_cast<uint2*>(o_planes + Tp * nq * 128 + off) =
        make_uint2(pack_bf16x2(lf[0], lf[1]), pack_bf16x2(lf[2], lf[3]));
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, m);
  if (lane == 0) {
    const long long b = row / S, t = row % S;
    delta[(b * nq + h) * stride + t] = dl;
  }
}

// ------------------------------------------------------------------ attention backward --
// A CTA per (64-key block j, KV group g, sequence b). For each query head h of the group and each
// 64-query block i >= j: S = scale q_i k_j^T, P = exp(S - lse) (causal), dV_j += P^T dO_i,
// dP = dO_i v_j^T, dS = P o (dP - delta), dK_j += scale dS^T q_i, dQ_i += scale dS k_j (atomic).
constexpr int AB = 64;  // keys and queries per block

template <typename Tl>
__global__ void __launch_bounds__(256) attn_bwd_kernel(const Tl* __restrict__ q, const Tl* __restrict__ k,
                                                       const Tl* __restrict__ v, const float* __restrict__ dO,
                                                       const float* __restrict__ lse, const float* __restrict__ delta,
                                                       float* __restrict__ dq, float* __restrict__ dk,
                                                       float* __restrict__ dv, int S, int nq, int nkv, int d,
                                                       float scale) {
  extern __shared__ float sb[];
  const int D = d, DP = d + 1;  // padded rows: the rows a warp reads at one column fall in different banks
  float* ks = sb;                // [AB][DP]
  float* vs = ks + AB * DP;      // [AB][DP]
  float* qs = vs + AB * DP;      // [AB][DP]
  float* dos = qs + AB * DP;     // [AB][DP]
  float* ps = dos + AB * DP;     // [AB][AB + 1] P
  float* dps = ps + AB * (AB + 1);  // [AB][AB + 1] dP
  float* ls = dps + AB * (AB + 1);  // [AB] lse
  float* ds_ = ls + AB;             // [AB] delta
  const int j = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = nq / nkv, Lq = nq * d, Lkv = nkv * d;
  const long long rb = (long long)b * S;
  const int k0 = j * AB;
  if (k0 >= S) return;
  const int tid = threadIdx.x;
  for (int e = tid; e < AB * D; e += 256) {
    const int r = e / D, c = e % D;
    const bool ok = k0 + r < S;
    ks[r * DP + c] = ok ? ld_f(k + (rb + k0 + r) * Lkv + g * d + c) : 0.f;
    vs[r * DP + c] = ok ? ld_f(v + (rb + k0 + r) * Lkv + g * d + c) : 0.f;
  }
  // dK_j and dV_j: thread owns (row r = tid / 4, columns c = (tid % 4) + 4 u) for u < D / 4
  const int orow = tid >> 2, ocol = tid & 3;
  float dka[32], dva[32];
#pragma unroll
  for (int u = 0; u < 32; ++u) dka[u] = dva[u] = 0.f;
  __syncthreads();
  for (int hh = 0; hh < G; ++hh) {
    const int h = g * G + hh;
    for (int q0 = k0; q0 < S; q0 += AB) {
      for (int e = tid; e < AB * D; e += 256) {
        const int r = e / D, c = e % D;
        const bool ok = q0 + r < S;
        qs[r * DP + c] = ok ? ld_f(q + (rb + q0 + r) * Lq + h * d + c) : 0.f;
        dos[r * DP + c] = ok ? dO[(rb + q0 + r) * Lq + h * d + c] : 0.f;
      }
      for (int r = tid; r < AB; r += 256) {
        const bool ok = q0 + r < S;
        ls[r] = ok ? lse[(rb + q0 + r) * nq + h] : 0.f;
        ds_[r] = ok ? delta[(rb + q0 + r) * nq + h] : 0.f;
      }
      __syncthreads();
      // P and dP: thread computes a 4 x 4 patch (query rows qr*4.., key cols kc*4..)
      {
        const int qr = tid / 16, kc = tid % 16;
        float sacc[4][4] = {}, pacc[4][4] = {};
        for (int c = 0; c < D; ++c) {
          float qa[4], da[4], kb[4], vb[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            qa[i] = qs[(qr * 4 + i) * DP + c];
            da[i] = dos[(qr * 4 + i) * DP + c];
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            kb[i] = ks[(kc * 4 + i) * DP + c];
            vb[i] = vs[(kc * 4 + i) * DP + c];
          }
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
              sacc[a][bb] = fmaf(qa[a], kb[bb], sacc[a][bb]);
              pacc[a][bb] = fmaf(da[a], vb[bb], pacc[a][bb]);
            }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int bb = 0; bb < 4; ++bb) {
            const int qi = qr * 4 + a, kj = kc * 4 + bb;
            const bool vis = q0 + qi < S && k0 + kj < S && k0 + kj <= q0 + qi;
            const float p = vis ? expf(sacc[a][bb] * scale - ls[qi]) : 0.f;
            ps[qi * (AB + 1) + kj] = p;
            dps[qi * (AB + 1) + kj] = p * (pacc[a][bb] - ds_[qi]);  // dS (before the scale)
          }
      }
      __syncthreads();
      // dV_j += P^T dO_i, dK_j += scale dS^T q_i
      for (int qi = 0; qi < AB; ++qi) {
        const float p = ps[qi * (AB + 1) + orow], dsv = dps[qi * (AB + 1) + orow];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const int c = ocol + 4 * u;
          if (c < D) {
            dva[u] = fmaf(p, dos[qi * DP + c], dva[u]);
            dka[u] = fmaf(dsv * scale, qs[qi * DP + c], dka[u]);
          }
        }
      }
      // dQ_i += scale dS k_j: thread (row qi = tid / 4, columns ocol + 4u)
      {
        const int qi = orow;
        if (q0 + qi < S) {
          float acc[32];
#pragma unroll
          for (int u = 0; u < 32; ++u) acc[u] = 0.f;
          for (int kj = 0; kj < AB; ++kj) {
            const float dsv = dps[qi * (AB + 1) + kj] * scale;
#pragma unroll
            for (int u = 0; u < 32; ++u) {
              const int c = ocol + 4 * u;
              if (c < D) acc[u] = fmaf(dsv, ks[kj * DP + c], acc[u]);
            }
          }
          float* dqr = dq + (rb + q0 + qi) * Lq + h * d;
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const int c = ocol + 4 * u;
            if (c < D) atomicAdd(dqr + c, acc[u]);
          }
        }
      }
      __syncthreads();
    }
  }
  if (k0 + orow < S) {
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int c = ocol + 4 * u;
      if (c < D) {
        dk[(rb + k0 + orow) * Lkv + g * d + c] = dka[u];
        dv[(rb + k0 + orow) * Lkv + g * d + c] = dva[u];
      }
    }
  }
}

// Where the latents' gradient goes: fp32 [T, Nlat] (f32), or for the tensor-core GEMMs its bf16 pair
// hi = bf16(v), lo = bf16(v - hi) twice: row-major [T][hi Nlat | lo Nlat] (rm, the dx GEMM's K-major
// operand) and as two planes [2][Tp][Nlat] (planes, the weight-gradient GEMMs' MN-major operand).
struct DlatOut {
  float* f32;
  __nv_bfloat16* rm;
  __nv_bfloat16* planes;
  int Nlat;
  long long Tp;
};

__device__ __forceinline__ void store_dlat(const DlatOut& o, long long row, int col, float v) {
  if (o.f32 != nullptr) {
    o.f32[row * o.Nlat + col] = v;
  } else {
    const __nv_bfloat16 hi = __float2bfloat16_rn(v), lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    o.rm[row * 2 * o.Nlat + col] = hi;
    o.rm[row * 2 * o.Nlat + o.Nlat + col] = lo;
    o.planes[row * o.Nlat + col] = hi;
    o.planes[(o.Tp + row) * o.Nlat + col] = lo;
  }
}

// ------------------------------------------------------------------ per-token backward --
// Row t of one sequence: dq, dk turned back by RoPE; the QK-mean transpose gives dc (the
// channel-mix outputs' gradient) and the latents' direct gradient dpre; dv goes through the value
// shift's transpose (channels [vfrom, Lkv) take the next token's gradient). A block takes two rows,
// 128 threads each. Thread = one pair (i, i + d/2) of one KV group g: the group's G query heads and
// its K head are turned by the same angle t theta_i (one sincos), and the QK-mean terms of the
// group's channels i and i + d/2 need only those heads. Then one V channel per thread and step.
struct Theta64 {
  double v[64];  // base^(-2i/d)
};

__device__ __forceinline__ void rope_back(float& x1, float& x2, float cs, float sn) {
  const float y1 = x1 * cs + x2 * sn, y2 = x2 * cs - x1 * sn;
  x1 = y1;
  x2 = y2;
}

__global__ void __launch_bounds__(256) token_bwd_kernel(const float* __restrict__ dq, const float* __restrict__ dk,
                                                        const float* __restrict__ dv, float* __restrict__ dc,
                                                        float* __restrict__ dpre, const DlatOut dlat, long long T,
                                                        int S, int nq, int nkv, int d, int mode, int vshift, int vfrom,
                                                        int use_rope, const __grid_constant__ Theta64 theta,
                                                        int plain) {
  const long long row = 2 * (long long)blockIdx.x + (threadIdx.x >> 7);  // b * S + t
  if (row >= T) return;
  const int lt = threadIdx.x & 127;
  const int t = (int)(row % S);
  const int G = nq / nkv, Lq = nq * d, Lkv = nkv * d, half = d / 2, W = Lq + Lkv;
  const float R = (mode & 1) ? 1.f : 0.f, P = (mode & 2) ? 1.f : 0.f;
  const float* dqr = dq + row * Lq;
  const float* dkr = dk + row * Lkv;
  for (int e = lt; e < nkv * half; e += 128) {
    const int g = e / half, i = e % half;
    float cs = 1.f, sn = 0.f;
    if (use_rope) {  // turn back by t theta_i (angle reduced in fp64)
      const double a = (double)t * theta.v[i];
      const double kk = rint(a * 0.15915494309189535);
      double r = fma(-kk, 6.283185307179586, a);
      r = fma(-kk, 2.4492935982947064e-16, r);
      sincosf((float)r, &sn, &cs);
    }
    float k1 = dkr[g * d + i], k2 = dkr[g * d + i + half];
    if (use_rope) rope_back(k1, k2, cs, sn);
    // QK-mean transpose: da_h = dqa_h / 2 + dka_g / (2G), db_g = sum_{h in g} dqa_h / 2 + dka_g / 2
    float s1 = 0.f, s2 = 0.f;
    for (int hh = 0; hh < G; ++hh) {
      const int c = (g * G + hh) * d + i;
      float q1 = dqr[c], q2 = dqr[c + half];
      if (use_rope) rope_back(q1, q2, cs, sn);
      s1 += q1;
      s2 += q2;
      const float a1 = 0.5f * q1 + (0.5f / (float)G) * k1, a2 = 0.5f * q2 + (0.5f / (float)G) * k2;
      if (plain) {  // no convolutions: the attention inputs are the latents
        store_dlat(dlat, row, c, q1);
        store_dlat(dlat, row, c + half, q2);
      } else {
        dc[row * W + c] = q1 + P * a1;
        dc[row * W + c + half] = q2 + P * a2;
        dpre[row * W + c] = R * a1;
        dpre[row * W + c + half] = R * a2;
      }
    }
    const int c = Lq + g * d + i;
    const float a1 = 0.5f * s1 + 0.5f * k1, a2 = 0.5f * s2 + 0.5f * k2;
    if (plain) {
      store_dlat(dlat, row, c, k1);
      store_dlat(dlat, row, c + half, k2);
    } else {
      dc[row * W + c] = k1 + P * a1;
      dc[row * W + c + half] = k2 + P * a2;
      dpre[row * W + c] = R * a1;
      dpre[row * W + c + half] = R * a2;
    }
  }
  // value shift transpose
  for (int c = lt; c < Lkv; c += 128) {
    float val;
    if (vshift && c >= vfrom) val = (t + 1 < S) ? dv[(row + 1) * Lkv + c] : 0.f;
    else val = dv[row * Lkv + c];
    store_dlat(dlat, row, Lq + Lkv + c, val);
  }
}

// Channel-mix backward of one head over a block of rows: ds[t] = W_c^T dc[t] and the block's share
// of dW_c = sum_t dc[t]^T s[t], s being the seq-conv output recomputed from the latents. A CTA per
// (CM_ROWS-row block, head; q heads then K heads), head_dim 128: W_c in shared memory, then 32-row
// sub-blocks of dc (row-major and transposed) and s; each thread owns 4 x 4 outputs of ds and an
// 8 x 8 patch of dW_c, added to the fp32 sum with vector atomics at the end.
constexpr int CM_ROWS = 256, CM_SUB = 32, CM_D = 128, CM_KMAX = 8;
constexpr size_t CM_SMEM = sizeof(float) * ((size_t)CM_D * CM_D + 2 * CM_SUB * CM_D + CM_D * (CM_SUB + 4) +
                                            (size_t)(CM_SUB + CM_KMAX - 1) * CM_D + CM_D * CM_KMAX + CM_SUB);

template <typename Tl, typename Tc>
__global__ void __launch_bounds__(256) chanmix_bwd_kernel(const float* __restrict__ dc, const Tl* __restrict__ lat,
                                                          const Tc* __restrict__ cq_chan, const Tc* __restrict__ ck_chan,
                                                          const Tc* __restrict__ cq_seq, const Tc* __restrict__ ck_seq,
                                                          float* __restrict__ ds, float* __restrict__ dwq,
                                                          float* __restrict__ dwk, long long T, int S, int nq, int nkv,
                                                          int K) {
  extern __shared__ float cm[];
  float* Wc = cm;                         // [i][j]
  float* dcR = Wc + CM_D * CM_D;          // [t][i]
  float* sR = dcR + CM_SUB * CM_D;        // [t][j]
  float* dcT = sR + CM_SUB * CM_D;        // [i][t] (row stride CM_SUB + 4)
  constexpr int LT = CM_SUB + 4;
  float* latS = dcT + CM_D * LT;          // [K - 1 + CM_SUB rows][CM_D]: latents of the sub-block and its halo
  float* wS = latS + (CM_SUB + CM_KMAX - 1) * CM_D;  // [c][k] seq-conv taps of the head
  int* tsS = reinterpret_cast<int*>(wS + CM_D * CM_KMAX);  // [t] position of each row in its sequence
  const int h = blockIdx.y, tid = threadIdx.x;
  const bool isq = h < nq;
  const int hh = isq ? h : h - nq;
  const int Lq = nq * CM_D, W = Lq + nkv * CM_D, Nlat = Lq + 2 * nkv * CM_D;
  const int ccol = isq ? hh * CM_D : Lq + hh * CM_D;  // this head's first column in dc / ds / lat
  const Tc* wsrc = (isq ? cq_chan : ck_chan) + (size_t)hh * CM_D * CM_D;
  const Tc* wseq = (isq ? cq_seq : ck_seq) + (size_t)hh * CM_D * K;
  for (int e = tid; e < CM_D * CM_D; e += 256) Wc[e] = ld_f(wsrc + e);
  for (int e = tid; e < CM_D * K; e += 256) wS[e] = ld_f(wseq + e);
  const int rq = tid >> 5, cq = tid & 31;  // ds: rows 4 rq .. +3, columns 4 cq .. +3
  const int pi = tid >> 4, pj = tid & 15;  // dW: rows 8 pi .. +7, columns 8 pj .. +7
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
  const long long r_begin = (long long)blockIdx.x * CM_ROWS;
  const long long r_end = r_begin + CM_ROWS < T ? r_begin + CM_ROWS : T;
  for (long long r0 = r_begin; r0 < r_end; r0 += CM_SUB) {
    __syncthreads();  // the previous sub-block's tiles are consumed (and Wc, wS are in place)
    // dc rows (four columns a thread) and the latent rows r0 - (K-1) .. r0 + CM_SUB - 1
    for (int e = tid; e < CM_SUB * (CM_D / 4); e += 256) {
      const int t = e / (CM_D / 4), c = 4 * (e % (CM_D / 4));
      const long long row = r0 + t;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (row < r_end) v = *reinterpret_cast<const float4*>(dc + row * W + ccol + c);
      *reinterpret_cast<float4*>(dcR + t * CM_D + c) = v;
    }
    if (tid < CM_SUB) tsS[tid] = (int)((r0 + tid) % S);
    for (int e = tid; e < (CM_SUB + K - 1) * CM_D; e += 256) {
      const int i = e / CM_D, c = e % CM_D;
      const long long row = r0 - (K - 1) + i;
      latS[i * CM_D + c] = (row >= 0 && row < r_end) ? ld_f(lat + row * Nlat + ccol + c) : 0.f;
    }
    __syncthreads();
    // s = the seq conv of the latents within each sequence (taps before a sequence start read
    // nothing), and dc transposed (a warp's stores spread over eight banks)
    for (int e = tid; e < CM_SUB * CM_D; e += 256) {
      const int t = e / CM_D, c = e % CM_D;
      dcT[c * LT + t] = dcR[t * CM_D + c];
      const int ts = tsS[t];
      float sv = 0.f;
      for (int k = 0; k < K; ++k)
        if (ts - (K - 1) + k >= 0) sv = fmaf(wS[c * K + k], latS[(t + k) * CM_D + c], sv);
      sR[t * CM_D + c] = sv;
    }
    __syncthreads();
    // ds = dc W_c: ds[t][j] = sum_i dc[t][i] W[i][j]
    {
      float o[4][4] = {};
#pragma unroll 4
      for (int i = 0; i < CM_D; ++i) {
        const float4 av = *reinterpret_cast<const float4*>(dcT + i * LT + 4 * rq);
        const float4 bv = *reinterpret_cast<const float4*>(Wc + i * CM_D + 4 * cq);
        const float a4[4] = {av.x, av.y, av.z, av.w}, b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) o[a][b] = fmaf(a4[a], b4[b], o[a][b]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const long long row = r0 + 4 * rq + a;
        if (row < r_end)
          *reinterpret_cast<float4*>(ds + row * W + ccol + 4 * cq) = make_float4(o[a][0], o[a][1], o[a][2], o[a][3]);
      }
    }
    // dW[i][j] += sum_t dc[t][i] s[t][j]
#pragma unroll 2
    for (int t = 0; t < CM_SUB; ++t) {
      const float4 a0 = *reinterpret_cast<const float4*>(dcR + t * CM_D + 8 * pi);
      const float4 a1 = *reinterpret_cast<const float4*>(dcR + t * CM_D + 8 * pi + 4);
      const float4 b0 = *reinterpret_cast<const float4*>(sR + t * CM_D + 8 * pj);
      const float4 b1 = *reinterpret_cast<const float4*>(sR + t * CM_D + 8 * pj + 4);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
    }
  }
  float* dw = (isq ? dwq : dwk) + (size_t)hh * CM_D * CM_D;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    float* rowp = dw + (size_t)(8 * pi + a) * CM_D + 8 * pj;
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(rowp), "f"(acc[a][0]), "f"(acc[a][1]),
                 "f"(acc[a][2]), "f"(acc[a][3])
                 : "memory");
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(rowp + 4), "f"(acc[a][4]), "f"(acc[a][5]),
                 "f"(acc[a][6]), "f"(acc[a][7])
                 : "memory");
  }
}

// The same for any even head_dim: per row t, per head, ds[t] = W_c^T dc[t] and s[t] recomputed
// (block = one row; thread = one channel); dW_c then comes from a strided GEMM over the rows.
template <typename Tl, typename Tc>
__global__ void __launch_bounds__(256) chan_bwd_kernel(const float* __restrict__ dc, const Tl* __restrict__ lat,
                                                       const Tc* __restrict__ cq_chan, const Tc* __restrict__ ck_chan,
                                                       const Tc* __restrict__ cq_seq, const Tc* __restrict__ ck_seq,
                                                       float* __restrict__ ds, float* __restrict__ s_out, int S,
                                                       int nq, int nkv, int d, int K) {
  const long long row = blockIdx.x;
  const int t = (int)(row % S);
  const int Lq = nq * d, Lkv = nkv * d, Nlat = Lq + 2 * Lkv, W = Lq + Lkv;
  for (int e = threadIdx.x; e < W; e += blockDim.x) {
    const bool isq = e < Lq;
    const int c = isq ? e : e - Lq;
    const int h = c / d, jj = c % d;
    const Tc* Wc = (isq ? cq_chan : ck_chan) + (long long)h * d * d;
    const float* dcr = dc + row * W + (isq ? 0 : Lq) + h * d;
    float acc = 0.f;
    for (int i = 0; i < d; ++i) acc = fmaf(ld_f(Wc + (long long)i * d + jj), dcr[i], acc);
    ds[row * W + e] = acc;
    const Tc* w = (isq ? cq_seq : ck_seq) + (long long)c * K;
    const int col = isq ? c : Lq + c;
    float sv = 0.f;
    for (int j = 0; j < K; ++j) {
      const int src = t - (K - 1) + j;
      if (src >= 0) sv = fmaf(ld_f(w + j), ld_f(lat + (row - t + src) * Nlat + col), sv);
    }
    s_out[row * W + e] = sv;
  }
}

// Seq-conv transpose and tap gradients in one pass over ds (both within each sequence):
//   dlat[t, c] = dpre[t, c] + sum_j w[c][j] ds[t + K-1-j, c]       (the q~ and k~ channels)
//   dw[c][j]   = sum_t ds[t, c] z[t - K+1 + j, c]                    (z: the latents)
// Thread = one channel over a slice of consecutive rows, with ds[t .. t+K-1] and z[t-K+1 .. t] in
// registers (one new row of each per step); block = 32 channels x 8 slices; the slices' tap sums
// reduce in shared memory, then atomically across blocks.
constexpr int kSeqSliceRows = 32;
template <int K, typename Tc, typename Tl>
__global__ void __launch_bounds__(256) seq_tap_bwd_kernel(const float* __restrict__ ds, const float* __restrict__ dpre,
                                                          const Tc* __restrict__ cq_seq, const Tc* __restrict__ ck_seq,
                                                          const Tl* __restrict__ lat, const DlatOut dlat,
                                                          float* __restrict__ dwq, float* __restrict__ dwk, long long T,
                                                          int S, int Lq, int Lkv) {
  __shared__ float red[8][32][K];
  const int W = Lq + Lkv, Nlat = Lq + 2 * Lkv;
  const int lane = threadIdx.x & 31, slice = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;  // latent column e (q~ channels, then k~)
  const long long r0 = ((long long)blockIdx.y * 8 + slice) * kSeqSliceRows;
  const long long r1 = r0 + kSeqSliceRows < T ? r0 + kSeqSliceRows : T;
  float acc[K];
#pragma unroll
  for (int j = 0; j < K; ++j) acc[j] = 0.f;
  if (e < W && r0 < T) {
    const Tc* wp = e < Lq ? cq_seq + (long long)e * K : ck_seq + (long long)(e - Lq) * K;
    float w[K], f[K], z[K];  // f[m] = ds[r + m], z[j] = z[r - K+1 + j]
#pragma unroll
    for (int j = 0; j < K; ++j) {
      w[j] = ld_f(wp + j);
      f[j] = 0.f;
      z[j] = 0.f;
    }
#pragma unroll
    for (int m = 0; m + 1 < K; ++m)
      if (r0 + m < T) f[m] = ds[(r0 + m) * W + e];
#pragma unroll
    for (int j = 0; j + 1 < K; ++j) {
      const long long src = r0 - (K - 1) + j;
      if (src >= 0) z[j] = ld_f(lat + src * Nlat + e);
    }
    int t = (int)(r0 % S);
#pragma unroll 1  // measured: unrolling 2 or 4 rows raised the registers and ran slower
    for (long long r = r0; r < r1; ++r) {
      f[K - 1] = r + K - 1 < T ? ds[(r + K - 1) * W + e] : 0.f;
      z[K - 1] = ld_f(lat + r * Nlat + e);
      float out = dpre[r * W + e];
#pragma unroll
      for (int j = 0; j < K; ++j)
        if (t + K - 1 - j < S) out = fmaf(w[j], f[K - 1 - j], out);
      store_dlat(dlat, r, e, out);
      const float g = f[0];
#pragma unroll
      for (int j = 0; j < K; ++j)
        if (t - (K - 1) + j >= 0) acc[j] = fmaf(g, z[j], acc[j]);
#pragma unroll
      for (int m = 0; m + 1 < K; ++m) {
        f[m] = f[m + 1];
        z[m] = z[m + 1];
      }
      if (++t == S) t = 0;
    }
  }
#pragma unroll
  for (int j = 0; j < K; ++j) red[slice][lane][j] = acc[j];
  __syncthreads();
  if (slice == 0 && e < W) {
#pragma unroll
    for (int j = 0; j < K; ++j) {
      float sum = 0.f;
      for (int sl = 0; sl < 8; ++sl) sum += red[sl][lane][j];
      float* dst = e < Lq ? dwq + (long long)e * K + j : dwk + (long long)(e - Lq) * K + j;
      atomicAdd(dst, sum);
    }
  }
}

template <int K, typename Tc, typename Tl>
cudaError_t launch_seq_tap_k(const float* ds, const float* dpre, const void* cq_seq, const void* ck_seq, const void* lat,
                             const DlatOut& dlat, float* dwq, float* dwk, long long T, int S, int Lq, int Lkv,
                             cudaStream_t stream) {
  const dim3 grid((unsigned)((Lq + Lkv + 31) / 32), (unsigned)((T + 8 * kSeqSliceRows - 1) / (8 * kSeqSliceRows)));
  seq_tap_bwd_kernel<K, Tc, Tl><<<grid, 256, 0, stream>>>(ds, dpre, static_cast<const Tc*>(cq_seq),
                                                          static_cast<const Tc*>(ck_seq), static_cast<const Tl*>(lat),
                                                          dlat, dwq, dwk, T, S, Lq, Lkv);
  return cudaGetLastError();
}

template <typename Tc, typename Tl>
cudaError_t launch_seq_tap(int K, const float* ds, const float* dpre, const void* cq_seq, const void* ck_seq,
                           const void* lat, const DlatOut& dlat, float* dwq, float* dwk, long long T, int S, int Lq,
                           int Lkv, cudaStream_t stream) {
  switch (K) {
#define CCA_SEQ_TAP_CASE(k) \
  case k:                   \
    return launch_seq_tap_k<k, Tc, Tl>(ds, dpre, cq_seq, ck_seq, lat, dlat, dwq, dwk, T, S, Lq, Lkv, stream);
    CCA_SEQ_TAP_CASE(1)
    CCA_SEQ_TAP_CASE(2)
    CCA_SEQ_TAP_CASE(3)
    CCA_SEQ_TAP_CASE(4)
    CCA_SEQ_TAP_CASE(5)
    CCA_SEQ_TAP_CASE(6)
    CCA_SEQ_TAP_CASE(7)
    CCA_SEQ_TAP_CASE(8)
#undef CCA_SEQ_TAP_CASE
    default:
      return cudaErrorInvalidValue;
  }
}

// Operands of the tensor-core GEMMs are bf16. A value v that bf16 does not hold exactly is carried as
// the pair hi = bf16(v), lo = bf16(v - hi) (about 16 significant bits, bf16's exponent range), laid
// side by side along the contraction so that one GEMM with a K two or three times longer sums
// hi*b + lo*b; the other operand, stored once, repeats along K (the GEMM's K wrap) ("Leveraging the
// bfloat16 artificial intelligence datatype for higher-precision computations", Henry et al., 2019).
enum SegKind : int { kSegNone = 0, kSegHi = 1, kSegLo = 2 };
struct Segs {
  int kind[3];
  long long off[3];  // element offset of each segment along the contraction
};
constexpr Segs kOneHi = {{kSegHi, kSegNone, kSegNone}, {0, 0, 0}};
__host__ __device__ constexpr Segs segs2(int k0, int k1, long long off1) { return {{k0, k1, kSegNone}, {0, off1, 0}}; }
__host__ __device__ constexpr Segs segs3(int k0, int k1, int k2, long long off) {
  return {{k0, k1, k2}, {0, off, 2 * off}};
}

__device__ __forceinline__ __nv_bfloat16 seg_value(float v, int kind) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  return kind == kSegLo ? __float2bfloat16_rn(v - __bfloat162float(hi)) : hi;
}

// Transposed: out[c * ldo + seg.off + r] = segment of in[r * ldi + c] for r < R, zero for R <= r < Rp
// (the padding of a contraction dimension). Row-major (rm non-null): rm[r * ldrm + rseg.off + c]. 32 x 32
// tiles through shared memory; rows of `in` run along grid x.
template <typename Ti>
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const Ti* __restrict__ in, long long ldi, int R, int C,
                                                             int Rp, __nv_bfloat16* __restrict__ out, long long ldo,
                                                             Segs seg, __nv_bfloat16* __restrict__ rm, long long ldrm,
                                                             Segs rseg) {
  __shared__ float tile[32][33];
  const long long r0 = (long long)blockIdx.x * 32;
  const int c0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int i = ty; i < 32; i += 8) {
    const long long r = r0 + i;
    const int c = c0 + tx;
    float v = 0.f;
    if (r < R && c < C) {
      v = ld_f(in + r * ldi + c);
      if (rm != nullptr) {
#pragma unroll
        for (int k = 0; k < 3; ++k)
          if (rseg.kind[k] != kSegNone) rm[r * ldrm + rseg.off[k] + c] = seg_value(v, rseg.kind[k]);
      }
    }
    tile[i][tx] = v;
  }
  __syncthreads();
  if (out == nullptr) return;
  for (int i = ty; i < 32; i += 8) {
    const int c = c0 + i;
    const long long r = r0 + tx;
    if (c < C && r < Rp) {
      const float v = tile[tx][i];
#pragma unroll
      for (int k = 0; k < 3; ++k)
        if (seg.kind[k] != kSegNone) out[(long long)c * ldo + seg.off[k] + r] = seg_value(v, seg.kind[k]);
    }
  }
}

cudaError_t transpose_bf16(Mat in, long long ldi, int R, int C, int Rp, __nv_bfloat16* out, long long ldo, Segs seg,
                           __nv_bfloat16* rm = nullptr, long long ldrm = 0, Segs rseg = kOneHi,
                           cudaStream_t s = 0) {
  const dim3 grid((unsigned)((Rp + 31) / 32), (unsigned)((C + 31) / 32));
  switch (in.t) {
    case DType::F32:
      transpose_bf16_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(in.p), ldi, R, C, Rp, out, ldo, seg,
                                                        rm, ldrm, rseg);
      break;
    case DType::BF16:
      transpose_bf16_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(in.p), ldi, R, C, Rp,
                                                                 out, ldo, seg, rm, ldrm, rseg);
      break;
    case DType::F16:
      transpose_bf16_kernel<__half><<<grid, 256, 0, s>>>(static_cast<const __half*>(in.p), ldi, R, C, Rp, out, ldo,
                                                         seg, rm, ldrm, rseg);
      break;
  }
  return cudaGetLastError();
}

// How the tcgen05 GEMM reads an operand: K wrap period and the K it holds (0: K), MN-major layout
// ([K][M or N]) and its row stride (0: dense)
struct Opnd {
  int kwrap = 0, kext = 0, mn = 0;
  long long ld = 0;
};
Opnd wrap(int period) {
  Opnd o;
  o.kwrap = period;
  return o;
}

// C[M, N] (fp32, row stride ldc, contiguous rows) = A[M, K] B[N, K]^T on the tensor cores, bf16
// operands; a long K over few output tiles is split (C cleared, slices added)
cudaError_t gemm_tc_bf16(const void* A, long long M, const void* B, int N, int K, float* C, long long ldc,
                         unsigned* err, cudaStream_t s, Opnd ao = Opnd(), Opnd bo = Opnd()) {
  GemmTcArgs a{};
  a.a_kwrap = ao.kwrap;
  a.a_kext = ao.kext;
  a.a_mn = ao.mn;
  a.lda = ao.ld;
  a.b_kwrap = bo.kwrap;
  a.b_kext = bo.kext;
  a.b_mn = bo.mn;
  a.ldb = bo.ld;
  a.ksplit = gemm_tc_ksplit(M, N, K);
  if (a.ksplit > 1) {
    const cudaError_t e = cudaMemsetAsync(C, 0, sizeof(float) * ((size_t)(M - 1) * ldc + N), s);
    if (e != cudaSuccess) return e;
  }
  a.A = A;
  a.M = M;
  a.K = K;
  a.B[0] = B;
  a.nrows[0] = N;
  a.nb = 1;
  a.C = C;
  a.ldc = ldc;
  a.in = DType::BF16;
  a.out = DType::F32;
  a.dev_err = err;
  return launch_gemm_tc(a, s);
}

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

bool backward_supported(const BlockDims& dm) {
  // the per-token kernel keeps one row's q and K gradients in shared memory
  return dm.K >= 0 && dm.K <= 8 && dm.d <= 128 && dm.d % 2 == 0 && dm.Lq + dm.Lkv <= 12288 &&
         ((dm.io == DType::BF16 && dm.lat == DType::F16) || (dm.io == DType::F32 && dm.lat == DType::F32));
}

// Workspace of the backward pass after the forward's own layout: the forward's outputs y, k_cache,
// v_cache (recomputed), then the fp32 buffers below.
BackwardLayout backward_layout(const BlockDims& dm, size_t forward_bytes) {
  BackwardLayout L;
  const size_t f = sizeof(float), T = (size_t)dm.T, W = (size_t)dm.Lq + dm.Lkv;
  size_t off = up256(forward_bytes);
  L.y = off;
  off = up256(off + T * dm.E * dtype_bytes(dm.out));
  L.k_cache = off;
  off = up256(off + T * dm.Lkv * dtype_bytes(dm.io));
  L.v_cache = off;
  off = up256(off + T * dm.Lkv * dtype_bytes(dm.io));
  L.stat_stride = (dm.S + 127) / 128 * 128;
  const size_t stats = (size_t)dm.B * dm.nq * L.stat_stride;  // >= T * nq, the SIMT path's layout
  L.dO = off;
  off = up256(off + f * T * dm.Lq);
  L.dO16 = off;
  off = up256(off + 2 * T * dm.Lq);
  L.lse = off;
  off = up256(off + f * stats);
  L.delta = off;
  off = up256(off + f * stats);
  L.dq = off;
  off = up256(off + f * T * dm.Lq);
  L.dk = off;
  off = up256(off + f * T * dm.Lkv);
  L.dv = off;
  off = up256(off + f * T * dm.Lkv);
  L.dc = off;
  off = up256(off + f * T * W);
  L.dpre = off;
  off = up256(off + f * T * W);
  L.ds = off;
  off = up256(off + f * T * W);
  L.s = off;
  off = up256(off + f * T * W);
  L.dlat = off;
  off = up256(off + f * T * dm.Nlat);
  // bf16 operands of the tensor-core GEMMs: transposed copies padded to Tp tokens (a multiple of the
  // GEMM's 64-deep K step), row-major copies, transposed weights
  L.Tp = (T + 63) / 64 * 64;
  const size_t h = 2, Tp = (size_t)L.Tp;
  // (segments along the contraction, see Segs)
  L.dy16 = off;
  off = up256(off + h * T * dm.E * 2);
  L.dy_t = off;
  off = up256(off + h * dm.E * Tp * 2);
  L.x_t = off;
  off = up256(off + h * dm.E * Tp);
  L.o_t = off;
  off = up256(off + h * dm.Lq * Tp * 3);
  L.dlat16 = off;
  off = up256(off + h * T * dm.Nlat * 2);
  L.dlat_t = off;
  off = up256(off + h * dm.Nlat * Tp * 2);
  L.wo_t = off;
  off = up256(off + h * dm.Lq * dm.E);
  L.w_t = off;
  off = up256(off + h * dm.E * dm.Nlat);
  L.dw_all = off;  // fp32 [Nlat, E]: the three weight gradients of the down-projection from one GEMM
  off = up256(off + f * dm.Nlat * dm.E);
  L.total = off;
  return L;
}

cudaError_t launch_backward(const BlockDims& dm, const BlockPtrs& p, const BackwardPtrs& g, const BackwardLayout& L,
                            char* ws, cudaStream_t stream, bool tc_attention, bool tc_gemm) {
  cudaError_t e;
  const long long T = dm.T;
  const int Lq = dm.Lq, Lkv = dm.Lkv, Nlat = dm.Nlat, E = dm.E, W = Lq + Lkv, d = dm.d;
  float* dO = reinterpret_cast<float*>(ws + L.dO);
  float* lse = reinterpret_cast<float*>(ws + L.lse);
  float* delta = reinterpret_cast<float*>(ws + L.delta);
  float* dq = reinterpret_cast<float*>(ws + L.dq);
  float* dk = reinterpret_cast<float*>(ws + L.dk);
  float* dv = reinterpret_cast<float*>(ws + L.dv);
  float* dc = reinterpret_cast<float*>(ws + L.dc);
  float* dpre = reinterpret_cast<float*>(ws + L.dpre);
  float* ds = reinterpret_cast<float*>(ws + L.ds);
  float* s = reinterpret_cast<float*>(ws + L.s);
  float* dlat = reinterpret_cast<float*>(ws + L.dlat);
  const DType lt = dm.lat, it = dm.io, ot = dm.out;
  const int Tp = L.Tp;
  __nv_bfloat16* dy16 = reinterpret_cast<__nv_bfloat16*>(ws + L.dy16);
  __nv_bfloat16* dy_t = reinterpret_cast<__nv_bfloat16*>(ws + L.dy_t);
  __nv_bfloat16* x_t = reinterpret_cast<__nv_bfloat16*>(ws + L.x_t);
  __nv_bfloat16* o_t = reinterpret_cast<__nv_bfloat16*>(ws + L.o_t);
  __nv_bfloat16* dlat16 = reinterpret_cast<__nv_bfloat16*>(ws + L.dlat16);
  __nv_bfloat16* dlat_t = reinterpret_cast<__nv_bfloat16*>(ws + L.dlat_t);
  __nv_bfloat16* wo_t = reinterpret_cast<__nv_bfloat16*>(ws + L.wo_t);
  __nv_bfloat16* w_t = reinterpret_cast<__nv_bfloat16*>(ws + L.w_t);
  // The tensor-core GEMMs read dy, x and W_o in place (MN-major where they are the transposed operand);
  // the latents' gradient and O come as bf16 hi / lo forms written by the kernels that make them.
  // An fp32 dy, or a block whose attention ran on the CUDA cores, takes bf16 copies made by transposes.
  const bool direct = tc_gemm && tc_attention && ot == DType::BF16;
  const long long TpLL = Tp;
  // 1. dO = dy W_o  [T, Lq];  dW_o = dy^T O  [E, Lq] (after step 2 on the direct path)
  if (direct) {
    Opnd wo;  // W_o [E][Lq] is [K][N]
    wo.mn = 1;
    wo.ld = Lq;
    if ((e = gemm_tc_bf16(g.dy, T, p.Wo, Lq, E, dO, Lq, p.dev_err, stream, Opnd(), wo)) != cudaSuccess) return e;
  } else if (tc_gemm) {
    // dO = dy W_o: exact bf16 products when dy is bf16; an fp32 dy is split in two segments
    // dW_o = dy^T O: O (fp16) is split, dy repeats over both segments; an fp32 dy is split too, with
    // the segments [hi, lo, hi] (dy repeating after two) x [hi, hi, lo] (three products)
    const bool dy_bf16 = ot == DType::BF16;
    const long long TpL = Tp;
    if ((e = transpose_bf16({p.Wo, it}, Lq, E, Lq, E, wo_t, E, kOneHi, nullptr, 0, kOneHi, stream)) != cudaSuccess)
      return e;
    if (dy_bf16) {
      if ((e = transpose_bf16({g.dy, ot}, E, (int)T, E, Tp, dy_t, TpL, kOneHi, nullptr, 0, kOneHi, stream)) !=
              cudaSuccess ||
          (e = transpose_bf16({p.o, lt}, Lq, (int)T, Lq, Tp, o_t, 2 * TpL, segs2(kSegHi, kSegLo, TpL), nullptr, 0,
                              kOneHi, stream)) != cudaSuccess)
        return e;
      if ((e = gemm_tc_bf16(g.dy, T, wo_t, Lq, E, dO, Lq, p.dev_err, stream)) != cudaSuccess ||
          (e = gemm_tc_bf16(dy_t, E, o_t, Lq, 2 * Tp, g.dWo, Lq, p.dev_err, stream, wrap(Tp))) != cudaSuccess)
        return e;
    } else {
      if ((e = transpose_bf16({g.dy, ot}, E, (int)T, E, Tp, dy_t, 2 * TpL, segs2(kSegHi, kSegLo, TpL), dy16, 2LL * E,
                              segs2(kSegHi, kSegLo, E), stream)) != cudaSuccess ||
          (e = transpose_bf16({p.o, lt}, Lq, (int)T, Lq, Tp, o_t, 3 * TpL, segs3(kSegHi, kSegHi, kSegLo, TpL), nullptr,
                              0, kOneHi, stream)) != cudaSuccess)
        return e;
      if ((e = gemm_tc_bf16(dy16, T, wo_t, Lq, 2 * E, dO, Lq, p.dev_err, stream, Opnd(), wrap(E))) != cudaSuccess ||
          (e = gemm_tc_bf16(dy_t, E, o_t, Lq, 3 * Tp, g.dWo, Lq, p.dev_err, stream, wrap(2 * Tp))) != cudaSuccess)
        return e;
    }
  } else {
    if ((e = gemm({g.dy, ot}, E, 1, 0, {p.Wo, it}, 1, Lq, 0, dO, Lq, 0, (int)T, Lq, E, 1, false, stream)) !=
        cudaSuccess)
      return e;
    if ((e = gemm({g.dy, ot}, 1, E, 0, {p.o, lt}, 1, Lq, 0, g.dWo, Lq, 0, E, Lq, T, 1, false, stream)) != cudaSuccess)
      return e;
  }
  if (tc_attention) {
    // 2. dO in fp16 and delta; the forward's tensor-core attention left lse2 (base 2)
    {
      const long long warps = T * dm.nq;
      do_prep_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, stream>>>(
          dO, static_cast<const __half*>(p.o), reinterpret_cast<__half*>(ws + L.dO16), delta, T, dm.S, dm.nq,
          L.stat_stride, direct ? o_t : nullptr, TpLL);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (direct) {
      // dW_o = dy^T [O_hi; O_lo]: dy read [T][E] as the MN-major A, repeating after Tp rows (T of them
      // held); O's two planes [2][Tp][Lq] as the MN-major B, their padding rows cleared
      for (int pl = 0; pl < 2 && Tp > T; ++pl)
        if ((e = cudaMemsetAsync(o_t + ((size_t)pl * Tp + T) * Lq, 0, sizeof(__nv_bfloat16) * (Tp - T) * Lq,
                                 stream)) != cudaSuccess)
          return e;
      Opnd dya, ob;
      dya.kwrap = Tp;
      dya.kext = (int)T;
      dya.mn = 1;
      dya.ld = E;
      ob.mn = 1;
      ob.ld = Lq;
      if ((e = gemm_tc_bf16(g.dy, E, o_t, Lq, 2 * Tp, g.dWo, Lq, p.dev_err, stream, dya, ob)) != cudaSuccess) return e;
    }
    // 3. attention backward on the tensor cores (dk, dv are sums over the CTAs of a key tile)
    if ((e = cudaMemsetAsync(dk, 0, sizeof(float) * T * Lkv, stream)) != cudaSuccess ||
        (e = cudaMemsetAsync(dv, 0, sizeof(float) * T * Lkv, stream)) != cudaSuccess)
      return e;
    AttnBwdPtrs a{p.q, p.k_att, p.v_att, ws + L.dO16, lse, delta, L.stat_stride, dq, dk, dv};
    if ((e = launch_attention_bwd_tc(dm, a, p.dev_err, stream)) != cudaSuccess) return e;
  } else {
    // 2. softmax statistics
    {
      const size_t smem = sizeof(float) * 2 * RB * (d + 1);
      const dim3 grid((dm.S + RB - 1) / RB, dm.nq, dm.B);
      if ((e = cudaFuncSetAttribute(row_stats_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
              cudaSuccess ||
          (e = cudaFuncSetAttribute(row_stats_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
              cudaSuccess)
        return e;
      if (lt == DType::F16)
        row_stats_kernel<__half><<<grid, 256, smem, stream>>>(static_cast<const __half*>(p.q),
                                                              static_cast<const __half*>(p.k_att),
                                                              static_cast<const __half*>(p.o), dO, lse, delta, dm.S,
                                                              dm.nq, dm.nkv, d, dm.scale);
      else
        row_stats_kernel<float><<<grid, 256, smem, stream>>>(static_cast<const float*>(p.q),
                                                             static_cast<const float*>(p.k_att),
                                                             static_cast<const float*>(p.o), dO, lse, delta, dm.S,
                                                             dm.nq, dm.nkv, d, dm.scale);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // 3. attention backward
    if ((e = cudaMemsetAsync(dq, 0, sizeof(float) * T * Lq, stream)) != cudaSuccess) return e;
    {
      const size_t smem = sizeof(float) * ((size_t)4 * AB * (d + 1) + 2 * AB * (AB + 1) + 2 * AB);
      const dim3 grid((dm.S + AB - 1) / AB, dm.nkv, dm.B);
      if (lt == DType::F16) {
        auto k = attn_bwd_kernel<__half>;
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
          return e;
        k<<<grid, 256, smem, stream>>>(static_cast<const __half*>(p.q), static_cast<const __half*>(p.k_att),
                                       static_cast<const __half*>(p.v_att), dO, lse, delta, dq, dk, dv, dm.S, dm.nq,
                                       dm.nkv, d, dm.scale);
      } else {
        auto k = attn_bwd_kernel<float>;
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
          return e;
        k<<<grid, 256, smem, stream>>>(static_cast<const float*>(p.q), static_cast<const float*>(p.k_att),
                                       static_cast<const float*>(p.v_att), dO, lse, delta, dq, dk, dv, dm.S, dm.nq,
                                       dm.nkv, d, dm.scale);
      }
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  // the latents' gradient: fp32, or (direct) its bf16 hi / lo forms with the planes' padding rows cleared
  DlatOut dlat_out{direct ? nullptr : dlat, dlat16, dlat_t, Nlat, TpLL};
  if (direct)
    for (int pl = 0; pl < 2 && Tp > T; ++pl)
      if ((e = cudaMemsetAsync(dlat_t + ((size_t)pl * Tp + T) * Nlat, 0, sizeof(__nv_bfloat16) * (Tp - T) * Nlat,
                               stream)) != cudaSuccess)
        return e;
  // 4. per-token: RoPE back, QK-mean transpose, value-shift transpose
  {
    Theta64 th{};
    for (int i = 0; i < d / 2; ++i) th.v[i] = pow((double)dm.rope_base, -2.0 * (double)i / (double)d);
    token_bwd_kernel<<<(unsigned)((T + 1) / 2), 256, 0, stream>>>(
        dq, dk, dv, dc, dpre, dlat_out, T, dm.S, dm.nq, dm.nkv, d, dm.qk_mean_mode, dm.value_shift, dm.vshift_from,
        dm.use_rope, th, dm.K == 0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (dm.K > 0) {
  // 5. channel mix: ds = W_c^T dc; dW_c[h] = sum_t dc[t,h]^T s[t,h] (s recomputed from the latents)
  if (tc_gemm && it == DType::BF16 && chanmix_bwd_tc_supported(dm)) {  // tensor cores (bf16 W_c is exact)
    if ((e = cudaMemsetAsync(g.dconvq_chan, 0, sizeof(float) * dm.nq * d * d, stream)) != cudaSuccess ||
        (e = cudaMemsetAsync(g.dconvk_chan, 0, sizeof(float) * dm.nkv * d * d, stream)) != cudaSuccess ||
        (e = launch_chanmix_bwd_tc(dm, dc, p.qkv_lat, p.cq_chan, p.ck_chan, p.cq_seq, p.ck_seq, ds, g.dconvq_chan,
                                   g.dconvk_chan, p.dev_err, stream)) != cudaSuccess)
      return e;
  } else if (d == CM_D) {
    if ((e = cudaMemsetAsync(g.dconvq_chan, 0, sizeof(float) * dm.nq * d * d, stream)) != cudaSuccess ||
        (e = cudaMemsetAsync(g.dconvk_chan, 0, sizeof(float) * dm.nkv * d * d, stream)) != cudaSuccess)
      return e;
    const dim3 grid((unsigned)((T + CM_ROWS - 1) / CM_ROWS), dm.nq + dm.nkv);
    if (lt == DType::F16 && it == DType::BF16) {
      auto k = chanmix_bwd_kernel<__half, __nv_bfloat16>;
      if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)CM_SMEM)) != cudaSuccess)
        return e;
      k<<<grid, 256, CM_SMEM, stream>>>(dc, static_cast<const __half*>(p.qkv_lat),
                                        static_cast<const __nv_bfloat16*>(p.cq_chan),
                                        static_cast<const __nv_bfloat16*>(p.ck_chan),
                                        static_cast<const __nv_bfloat16*>(p.cq_seq),
                                        static_cast<const __nv_bfloat16*>(p.ck_seq), ds, g.dconvq_chan, g.dconvk_chan, T,
                                        dm.S, dm.nq, dm.nkv, dm.K);
    } else {
      auto k = chanmix_bwd_kernel<float, float>;
      if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)CM_SMEM)) != cudaSuccess)
        return e;
      k<<<grid, 256, CM_SMEM, stream>>>(dc, static_cast<const float*>(p.qkv_lat), static_cast<const float*>(p.cq_chan),
                                        static_cast<const float*>(p.ck_chan), static_cast<const float*>(p.cq_seq),
                                        static_cast<const float*>(p.ck_seq), ds, g.dconvq_chan, g.dconvk_chan, T, dm.S,
                                        dm.nq, dm.nkv, dm.K);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else {
    if (lt == DType::F16 && it == DType::BF16)
      chan_bwd_kernel<__half, __nv_bfloat16><<<(unsigned)T, 256, 0, stream>>>(
          dc, static_cast<const __half*>(p.qkv_lat), static_cast<const __nv_bfloat16*>(p.cq_chan),
          static_cast<const __nv_bfloat16*>(p.ck_chan), static_cast<const __nv_bfloat16*>(p.cq_seq),
          static_cast<const __nv_bfloat16*>(p.ck_seq), ds, s, dm.S, dm.nq, dm.nkv, d, dm.K);
    else
      chan_bwd_kernel<float, float><<<(unsigned)T, 256, 0, stream>>>(
          dc, static_cast<const float*>(p.qkv_lat), static_cast<const float*>(p.cq_chan),
          static_cast<const float*>(p.ck_chan), static_cast<const float*>(p.cq_seq), static_cast<const float*>(p.ck_seq),
          ds, s, dm.S, dm.nq, dm.nkv, d, dm.K);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // dW_c (q heads, then K heads): batch over heads; A[i][t] = dc[t][h d + i], B[j][t] = s[t][h d + j]
    if ((e = gemm({dc, DType::F32}, 1, W, d, {s, DType::F32}, 1, W, d, g.dconvq_chan, d, (long long)d * d, d, d, T,
                  dm.nq, false, stream)) != cudaSuccess)
      return e;
    if ((e = gemm({dc + Lq, DType::F32}, 1, W, d, {s + Lq, DType::F32}, 1, W, d, g.dconvk_chan, d, (long long)d * d,
                  d, d, T, dm.nkv, false, stream)) != cudaSuccess)
      return e;
  }
  // 6. seq conv: dlat (q and k channels) and the tap gradients, one pass
  if ((e = cudaMemsetAsync(g.dconvq_seq, 0, sizeof(float) * Lq * dm.K, stream)) != cudaSuccess ||
      (e = cudaMemsetAsync(g.dconvk_seq, 0, sizeof(float) * Lkv * dm.K, stream)) != cudaSuccess)
    return e;
  e = it == DType::BF16 && lt == DType::F16
          ? launch_seq_tap<__nv_bfloat16, __half>(dm.K, ds, dpre, p.cq_seq, p.ck_seq, p.qkv_lat, dlat_out, g.dconvq_seq,
                                                  g.dconvk_seq, T, dm.S, Lq, Lkv, stream)
      : it == DType::F32 && lt == DType::F32
          ? launch_seq_tap<float, float>(dm.K, ds, dpre, p.cq_seq, p.ck_seq, p.qkv_lat, dlat_out, g.dconvq_seq,
                                         g.dconvk_seq, T, dm.S, Lq, Lkv, stream)
          : cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  }  // convolutions
  // 7. down-projection: dx = dlat [W_q; W_k; W_v];  dW_* = dlat^T x
  const void* Ws[3] = {p.Wq, p.Wk, p.Wv};
  float* dWs[3] = {g.dWq, g.dWk, g.dWv};
  const int col0[3] = {0, Lq, Lq + Lkv}, rows[3] = {Lq, Lkv, Lkv};
  if (direct) {
    // dx = [dlat_hi | dlat_lo] [W; W]: W^T (small) repeats over both segments; dW_* = [dlat_hi; dlat_lo]^T x:
    // the planes' columns of the weight as the MN-major A, x [T][E] as the MN-major B repeating after Tp
    for (int i = 0; i < 3; ++i)
      if ((e = transpose_bf16({Ws[i], it}, E, rows[i], E, rows[i], w_t + col0[i], Nlat, kOneHi, nullptr, 0, kOneHi,
                              stream)) != cudaSuccess)
        return e;
    if ((e = gemm_tc_bf16(dlat16, T, w_t, E, 2 * Nlat, g.dx, E, p.dev_err, stream, Opnd(), wrap(Nlat))) != cudaSuccess)
      return e;
    // one GEMM over all Nlat latent channels (four times the output tiles of the W_k or W_v share
    // alone) into fp32 scratch, then each weight's rows to its output
    Opnd la, xb;
    la.mn = 1;
    la.ld = Nlat;
    xb.kwrap = Tp;
    xb.kext = (int)T;
    xb.mn = 1;
    xb.ld = E;
    float* dW_all = reinterpret_cast<float*>(ws + L.dw_all);  // [Nlat, E]
    if ((e = gemm_tc_bf16(dlat_t, Nlat, p.x, E, 2 * Tp, dW_all, E, p.dev_err, stream, la, xb)) != cudaSuccess) return e;
    for (int i = 0; i < 3; ++i)
      if ((e = cudaMemcpyAsync(dWs[i], dW_all + (size_t)col0[i] * E, sizeof(float) * rows[i] * E,
                               cudaMemcpyDeviceToDevice, stream)) != cudaSuccess)
        return e;
    return cudaSuccess;
  }
  if (tc_gemm) {
    // dlat (fp32) split in two segments, row-major for dx and transposed for dW; x and the weights
    // are exact in bf16, stored once and repeated over both segments
    const long long TpL = Tp;
    if ((e = transpose_bf16({dlat, DType::F32}, Nlat, (int)T, Nlat, Tp, dlat_t, 2 * TpL, segs2(kSegHi, kSegLo, TpL),
                            dlat16, 2LL * Nlat, segs2(kSegHi, kSegLo, Nlat), stream)) != cudaSuccess ||
        (e = transpose_bf16({p.x, it}, E, (int)T, E, Tp, x_t, TpL, kOneHi, nullptr, 0, kOneHi, stream)) != cudaSuccess)
      return e;
    for (int i = 0; i < 3; ++i)
      if ((e = transpose_bf16({Ws[i], it}, E, rows[i], E, rows[i], w_t + col0[i], Nlat, kOneHi, nullptr, 0, kOneHi,
                              stream)) != cudaSuccess)
        return e;
    if ((e = gemm_tc_bf16(dlat16, T, w_t, E, 2 * Nlat, g.dx, E, p.dev_err, stream, Opnd(), wrap(Nlat))) !=
        cudaSuccess)
      return e;
    for (int i = 0; i < 3; ++i)
      if ((e = gemm_tc_bf16(dlat_t + (size_t)col0[i] * 2 * Tp, rows[i], x_t, E, 2 * Tp, dWs[i], E, p.dev_err, stream,
                            Opnd(), wrap(Tp))) != cudaSuccess)
        return e;
    return cudaSuccess;
  }
  for (int i = 0; i < 3; ++i) {
    // dx[t][e] (+)= sum_c dlat[t][col0 + c] W[c][e]
    if ((e = gemm({dlat + col0[i], DType::F32}, Nlat, 1, 0, {Ws[i], it}, 1, E, 0, g.dx, E, 0, (int)T, E, rows[i], 1,
                  i > 0, stream)) != cudaSuccess)
      return e;
    // dW[c][e] = sum_t dlat[t][col0 + c] x[t][e]
    if ((e = gemm({dlat + col0[i], DType::F32}, 1, Nlat, 0, {p.x, it}, 1, E, 0, dWs[i], E, 0, rows[i], E, T, 1, false,
                  stream)) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

}  // namespace cca
