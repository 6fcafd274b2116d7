// SIMT (CUDA-core, fp32 arithmetic) kernels: the general path for fp32 blocks
// and head dims the tensor-core kernels do not take.
//
//  * gemm_simt_kernel: C = A B^T with both operands K-contiguous (the
//    down-projection x W^T and the output projection o W_o^T of
//    "Compressed Convolutional Attention", es section 2.A).
//  * attention_simt_kernel: causal softmax attention on the compressed heads,
//    one K/V head per group of G query heads (es 2.A and 2.C), computed with
//    an online softmax over key tiles.
//  * convert_f16_kernel: an fp16 copy of a bf16 array (the intermediate-type copy of the
//    channel-conv weights when no tensor-core down-projection carries it as a side job).
#include <type_traits>

#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

constexpr int GT_M = 64, GT_N = 64, GT_K = 16;

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const Tin* __restrict__ A, long long lda,
                                                        const Tin* __restrict__ Bm, long long ldb,
                                                        Tout* __restrict__ C, long long ldc, long long M, int N,
                                                        int K, unsigned* err) {
  __shared__ float As[GT_K][GT_M + 4];
  __shared__ float Bs[GT_K][GT_N + 4];
  const int tid = threadIdx.x;
  const long long m0 = (long long)blockIdx.y * GT_M;
  const int n0 = blockIdx.x * GT_N;
  const int tr = tid / 16, tc = tid % 16;  // 16 x 16 threads, 4 x 4 outputs each
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += GT_K) {
    // 64 rows x 16 k per operand: 1024 elements, 4 per thread
    for (int e = tid; e < GT_M * GT_K; e += 256) {
      int r = e / GT_K, kk = e % GT_K;
      long long gm = m0 + r;
      int gk = k0 + kk;
      As[kk][r] = (gm < M && gk < K) ? ld_f(A + gm * lda + gk) : 0.f;
      int gn = n0 + r;
      Bs[kk][r] = (gn < N && gk < K) ? ld_f(Bm + (long long)gn * ldb + gk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < GT_K; ++kk) {
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
  float amax = 0.f;  // largest |C| stored, for the fp16 range report
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    long long gm = m0 + tr * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int gn = n0 + tc * 4 + j;
      if (gn < N) {
        st_f(C + gm * ldc + gn, acc[i][j]);
        amax = fmaxf(amax, fabsf(acc[i][j]));
      }
    }
  }
  if (std::is_same<Tout, __half>::value) report_range(amax > 65504.0f, err);
}

// Causal attention, SIMT. One CTA = 64 query rows of one query head; two
// threads per row, each owning half of the key tile in the score phase and
// half of the head dim in the output phase.
constexpr int AT_Q = 64, AT_K = 64;

template <typename T>
__global__ void __launch_bounds__(128) attention_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                             const T* __restrict__ v, T* __restrict__ o, int S,
                                                             int nq, int nkv, int d, float scale) {
  extern __shared__ float sm[];
  const int dp = d + 1;
  float* Qs = sm;                   // [AT_Q][d+1]
  float* Ks = Qs + AT_Q * dp;       // [AT_K][d+1]
  float* Vs = Ks + AT_K * dp;       // [AT_K][d]
  float* Ps = Vs + AT_K * d;        // [AT_Q][AT_K+1]
  const int tid = threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int G = nq / nkv, g = h / G;
  const int Lq = nq * d, Lkv = nkv * d;
  const int q0 = blockIdx.x * AT_Q;
  const long long rowbase = (long long)b * S;
  const int r = tid >> 1, half = tid & 1;
  const int dh = d / 2;

  for (int e = tid; e < AT_Q * d; e += 128) {
    int rr = e / d, i = e % d;
    int t = q0 + rr;
    Qs[rr * dp + i] = (t < S) ? ld_f(q + (rowbase + t) * Lq + (long long)h * d + i) : 0.f;
  }
  float m = -INFINITY, l = 0.f;
  float acc[64];
#pragma unroll
  for (int j = 0; j < 64; ++j) acc[j] = 0.f;
  const int tq = q0 + r;
  const int kend = min(S, q0 + AT_Q);  // keys [0, kend) can be seen by this tile
  for (int k0 = 0; k0 < kend; k0 += AT_K) {
    __syncthreads();
    for (int e = tid; e < AT_K * d; e += 128) {
      int rr = e / d, i = e % d;
      int s = k0 + rr;
      bool ok = s < S;
      long long off = (rowbase + s) * Lkv + (long long)g * d + i;
      Ks[rr * dp + i] = ok ? ld_f(k + off) : 0.f;
      Vs[rr * d + i] = ok ? ld_f(v + off) : 0.f;
    }
    __syncthreads();
    float sc[32];
    float tmax = -INFINITY;
#pragma unroll 4
    for (int c = 0; c < 32; ++c) {
      int kk = half * 32 + c;
      int s = k0 + kk;
      float dot = 0.f;
      for (int i = 0; i < d; ++i) dot = fmaf(Qs[r * dp + i], Ks[kk * dp + i], dot);
      float val = (s <= tq && s < S) ? dot * scale : -INFINITY;
      sc[c] = val;
      tmax = fmaxf(tmax, val);
    }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    const float mnew = fmaxf(m, tmax);
    // Rows past the sequence end see only masked keys in late tiles; keep them finite.
    const float mref = (mnew == -INFINITY) ? 0.f : mnew;
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - mref);
    float psum = 0.f;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      float p = (sc[c] == -INFINITY) ? 0.f : expf(sc[c] - mref);
      Ps[r * (AT_K + 1) + half * 32 + c] = p;
      psum += p;
    }
    psum += __shfl_xor_sync(0xffffffffu, psum, 1);
    l = l * alpha + psum;
    m = mnew;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 64; ++j)
      if (j < dh) acc[j] *= alpha;
    for (int kk = 0; kk < AT_K; ++kk) {
      float p = Ps[r * (AT_K + 1) + kk];
      const float* vrow = Vs + kk * d + half * dh;
#pragma unroll
      for (int j = 0; j < 64; ++j)
        if (j < dh) acc[j] = fmaf(p, vrow[j], acc[j]);
    }
  }
  if (tq < S) {
    const float inv = 1.f / l;
    T* orow = o + (rowbase + tq) * Lq + (long long)h * d + half * dh;
#pragma unroll
    for (int j = 0; j < 64; ++j)
      if (j < dh) st_f(orow + j, acc[j] * inv);
  }
}

}  // namespace

namespace {
template <typename Tin, typename Tout>
void gemm_simt_typed(const void* A, long long lda, const void* Bm, long long ldb, void* C, long long ldc,
                     long long M, int N, int K, unsigned* err, dim3 grid, cudaStream_t stream) {
  gemm_simt_kernel<Tin, Tout><<<grid, 256, 0, stream>>>((const Tin*)A, lda, (const Tin*)Bm, ldb, (Tout*)C, ldc, M,
                                                         N, K, err);
}
template <typename Tin>
void gemm_simt_out(DType out, const void* A, long long lda, const void* Bm, long long ldb, void* C, long long ldc,
                   long long M, int N, int K, unsigned* err, dim3 grid, cudaStream_t stream) {
  switch (out) {
    case DType::F32: gemm_simt_typed<Tin, float>(A, lda, Bm, ldb, C, ldc, M, N, K, err, grid, stream); break;
    case DType::BF16: gemm_simt_typed<Tin, __nv_bfloat16>(A, lda, Bm, ldb, C, ldc, M, N, K, err, grid, stream); break;
    case DType::F16: gemm_simt_typed<Tin, __half>(A, lda, Bm, ldb, C, ldc, M, N, K, err, grid, stream); break;
  }
}
}  // namespace

cudaError_t launch_gemm_simt(DType in, DType out, const void* A, long long lda, const void* Bm, long long ldb,
                             void* C, long long ldc, long long M, int N, int K, cudaStream_t stream,
                             unsigned* dev_err) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + GT_N - 1) / GT_N, (unsigned)((M + GT_M - 1) / GT_M));
  switch (in) {
    case DType::F32: gemm_simt_out<float>(out, A, lda, Bm, ldb, C, ldc, M, N, K, dev_err, grid, stream); break;
    case DType::BF16:
      gemm_simt_out<__nv_bfloat16>(out, A, lda, Bm, ldb, C, ldc, M, N, K, dev_err, grid, stream);
      break;
    case DType::F16: gemm_simt_out<__half>(out, A, lda, Bm, ldb, C, ldc, M, N, K, dev_err, grid, stream); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_attention_simt(const BlockDims& dm, const void* q, const void* k, const void* v, void* o,
                                  cudaStream_t stream) {
  const int d = dm.d;
  size_t smem = sizeof(float) * ((size_t)AT_Q * (d + 1) + (size_t)AT_K * (d + 1) + (size_t)AT_K * d +
                                 (size_t)AT_Q * (AT_K + 1));
  dim3 grid((dm.S + AT_Q - 1) / AT_Q, dm.nq, dm.B);
  cudaError_t e;
  if (dm.lat == DType::F16) {
    auto kern = attention_simt_kernel<__half>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
      return e;
    kern<<<grid, 128, smem, stream>>>((const __half*)q, (const __half*)k, (const __half*)v, (__half*)o, dm.S,
                                      dm.nq, dm.nkv, d, dm.scale);
  } else if (dm.lat == DType::F32) {
    auto kern = attention_simt_kernel<float>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
      return e;
    kern<<<grid, 128, smem, stream>>>((const float*)q, (const float*)k, (const float*)v, (float*)o, dm.S, dm.nq,
                                      dm.nkv, d, dm.scale);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

namespace {
__global__ void __launch_bounds__(256) convert_f16_kernel(const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst,
                                                          long long n, unsigned* err, float scale) {
  bool bad = false;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float f = __bfloat162float(src[i]) * scale;
    bad |= f16_overflow(f);
    dst[i] = __float2half_rn(f);
  }
  report_range(bad, err);
}
}  // namespace

cudaError_t launch_convert_f16(const void* src, void* dst, long long n, unsigned* dev_err, cudaStream_t stream,
                               float scale) {
  if (n <= 0) return cudaSuccess;
  long long blocks = (n + 255) / 256;
  if (blocks > 1184) blocks = 1184;
  convert_f16_kernel<<<(unsigned)blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(src),
                                                             static_cast<__half*>(dst), n, dev_err, scale);
  return cudaGetLastError();
}

}  // namespace cca
