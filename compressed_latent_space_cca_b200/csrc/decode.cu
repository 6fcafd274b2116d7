// One decode step of a CCA / CCGQA block: the token at position t = seq_len - 1 of each sequence,
// from the state a prefill (or earlier decode steps) left: KV-cache rows 0..t-1 and the conv state
// (the last K-1 pre-conv latents of q and k and the last v latent). The compressed cache is what
// decoding reads ("Compressed Convolutional Attention", gist.science/es/paper/2510.04476, section 1
// item 2; the cache is C times smaller than a multi-head one, section 4).
//
// Every step of the prefill runs for the one token in fp32 arithmetic (inputs, weights and cache in
// the block's type). A step is bound by moving the weights and the cache once, and at batch 1 by
// the latency of four dependent kernels, launched one after the other on the stream. The kernels
// can also run with programmatic dependent launch (each first issues the loads that do not depend
// on the kernel before it, then waits for it with griddepcontrol.wait); that form is switched off
// (kDecodePdl) because a run of the attention kernel under it produced a non-finite row whose cause
// was not found. The four kernels:
//   decode_down_kernel  z = x_t [W_q; W_k; W_v]^T: a warp per latent channel streams its weight row
//                       once and serves up to kGemvBatch sequences
//   decode_conv_kernel  a CTA per (head, KV group, sequence): the causal seq conv over the conv
//                       state and z, the head's channel mix, the shifted v row; then the conv state
//                       of the head's channels advances by one token
//   decode_attn_kernel  a CTA per (key chunk, KV group, sequence). Its key rows stream into a
//                       shared-memory ring (cp.async) from the start. Prologue: QK-mean and RoPE of
//                       the group's G query rows and of the new key (the chunk holding key t writes
//                       cache row t). Body: lanes split each key's head_dim, hold q in registers
//                       and keep an online softmax per head; the CTA's lane groups merge in shared
//                       memory, and the last chunk of a (group, sequence) to finish (an atomic
//                       count, no waiting) merges the chunks in two rounds of loads (every chunk's
//                       max and sum, then every chunk's output columns, a batch at a time)
//   decode_out_kernel   y_t = o W_o^T, a warp per output channel
// No kernel waits on a later one, so the chain always completes.
#include <math.h>

#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

constexpr int DNT = 256;           // threads of the GEMV and conv kernels
constexpr int ANT = 256;           // attention threads
constexpr int kGemvBatch = 8;      // sequences per GEMV launch
constexpr int kMaxChunks = 256;    // key chunks per (KV group, sequence)
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeArgs {
  const void *x, *Wq, *Wk, *Wv, *cq_seq, *cq_chan, *ck_seq, *ck_chan, *Wo;
  void *y, *k_cache, *v_cache, *conv_state;
  // workspace (fp32): z [B, Nlat] latents of the new token, c [B, Lq + Lkv] channel-mix outputs,
  // vt [B, Lkv] the new v row after the value shift, o [B, Lq] attention output, the chunks'
  // partial results part_o [B*nkv, nch, G, d] and part_ml [B*nkv, nch, G, 2] (max, sum), and one
  // finished-chunk counter per (sequence, KV group)
  float *z, *c, *vt, *o, *part_o, *part_ml;
  int* cnt;
  int B, E, nkv, d, K, G, Lq, Lkv, Nlat, t, rows, mode, vshift, vfrom, use_rope;
  int chunk_len, nch;  // keys per chunk, chunks per (KV group, sequence)
  float qscale;        // softmax scale * log2(e): scores in base-2 units
  float2 rot[64];      // (cos, sin) of t * base^(-2i/d), computed in double on the host
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// 16 bytes of a row: 8 bf16 or 4 fp32 elements
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static __forceinline__ void unpack(const uint4& u, float* v) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(h[k]);
      v[2 * k] = f.x;
      v[2 * k + 1] = f.y;
    }
  }
};
template <> struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static __forceinline__ void unpack(const uint4& u, float* v) {
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
  }
};
// 16-byte read-only load, issued where it stands: a volatile asm keeps the compiler from sinking
// a prefetch below the barrier or dependency wait that follows it
__device__ __forceinline__ uint4 ld16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// 16 bytes of Tc from 16 / sizeof(Tc) floats (round to nearest even)
__device__ __forceinline__ uint4 pack16(const float* v, __nv_bfloat16*) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
}
__device__ __forceinline__ uint4 pack16(const float* v, float*) {
  return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]));
}

// programmatic dependent launch: the next kernel in the stream may launch / wait until the previous
// kernel has completed and its writes are visible (a no-op for a kernel launched without it)
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// 16-byte asynchronous global -> shared copies, completed per commit group
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// One warp computes acc[b] = sum_e w[e] xs[b][e] for a row w of length n (a multiple of 8), b < nb,
// with xs in shared memory (fp32, or the weights' type). The lanes take consecutive 16-byte pieces
// of w; a batch of up to NL pieces per lane is in flight at once, and the caller may issue the
// row's first batch early (load) and pass it to run.
template <typename Tw, typename Tx>
struct RowDot {
  static constexpr int V = Vec16<Tw>::N;
  static constexpr int NL = 8;  // pieces per lane per batch
  __device__ static __forceinline__ void load(const Tw* w, int n, int base, uint4 (&r)[NL]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 0; k < NL; ++k) {
      const int e0 = base + (lane + 32 * k) * V;
      r[k] = e0 < n ? ld16(w + e0) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __device__ static __forceinline__ void xload(const float* xp, float (&v)[V]) {
#pragma unroll
    for (int q = 0; q < V; q += 4) {
      const float4 f = *reinterpret_cast<const float4*>(xp + q);
      v[q] = f.x, v[q + 1] = f.y, v[q + 2] = f.z, v[q + 3] = f.w;
    }
  }
  __device__ static __forceinline__ void xload(const __nv_bfloat16* xp, float (&v)[V]) {
    Vec16<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(xp), v);
  }
  __device__ static __forceinline__ void fma(const uint4 (&r)[NL], const Tx* xs, int n, int nb, int base,
                                             float (&acc)[kGemvBatch]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 0; k < NL; ++k) {
      const int e0 = base + (lane + 32 * k) * V;
      if (e0 < n) {
        float wv[V];
        Vec16<Tw>::unpack(r[k], wv);
#pragma unroll
        for (int b = 0; b < kGemvBatch; ++b) {
          if (b < nb) {
            float xv[V];
            xload(xs + b * n + e0, xv);
            float s = acc[b];
#pragma unroll
            for (int q = 0; q < V; ++q) s = fmaf(wv[q], xv[q], s);
            acc[b] = s;
          }
        }
      }
    }
  }
  __device__ static __forceinline__ void run(const Tw* w, int n, const Tx* xs, int nb, const uint4 (&first)[NL],
                                             float (&acc)[kGemvBatch]) {
    fma(first, xs, n, nb, 0, acc);
    for (int base = 32 * V * NL; base < n; base += 32 * V * NL) {
      uint4 r[NL];
      load(w, n, base, r);
      fma(r, xs, n, nb, base, acc);
    }
  }
};

// ---------------------------------------------------------------------------------------------
// z[b0 + b] = x_t[b0 + b] [W_q; W_k; W_v]^T for b < nb (es 2.A: the down-projection). The first
// kernel of a step: nothing in the step precedes it. x goes to shared memory asynchronously while
// the warp's first batch of weight pieces is in flight.
template <typename Tc>
__global__ void __launch_bounds__(DNT) decode_down_kernel(const __grid_constant__ DecodeArgs a, int b0, int nb) {
  using R = RowDot<Tc, Tc>;
  constexpr int V = R::V;
  pdl_launch_dependents();
  extern __shared__ __align__(16) unsigned char smd[];
  Tc* xs = reinterpret_cast<Tc*>(smd);  // [nb][E]
  const Tc* x = static_cast<const Tc*>(a.x) + (long long)b0 * a.E;
  for (int i = threadIdx.x * V; i < nb * a.E; i += DNT * V) cp_async16(xs + i, x + i);
  cp_async_commit();
  const int n = blockIdx.x * (DNT / 32) + (threadIdx.x >> 5);
  const Tc* w = nullptr;
  uint4 first[R::NL];
  if (n < a.Nlat) {
    w = n < a.Lq            ? static_cast<const Tc*>(a.Wq) + (long long)n * a.E
        : n < a.Lq + a.Lkv ? static_cast<const Tc*>(a.Wk) + (long long)(n - a.Lq) * a.E
                           : static_cast<const Tc*>(a.Wv) + (long long)(n - a.Lq - a.Lkv) * a.E;
    R::load(w, a.E, 0, first);
  }
  if (b0 == 0 && blockIdx.x == 0)
    for (int i = threadIdx.x; i < a.B * a.nkv; i += DNT) a.cnt[i] = 0;  // the attention's chunk counters
  cp_async_wait<0>();
  __syncthreads();
  if (n >= a.Nlat) return;
  float acc[kGemvBatch];
#pragma unroll
  for (int b = 0; b < kGemvBatch; ++b) acc[b] = 0.f;
  R::run(w, a.E, xs, nb, first, acc);
#pragma unroll
  for (int b = 0; b < kGemvBatch; ++b) {
    if (b < nb) {
      const float s = warp_sum(acc[b]);
      if ((threadIdx.x & 31) == 0) a.z[(long long)(b0 + b) * a.Nlat + n] = s;
    }
  }
}

// y_t[b0 + b] = o[b0 + b] W_o^T for b < nb. W_o's first batch is loaded before the wait for the
// attention kernel.
template <typename Tc, typename To>
__global__ void __launch_bounds__(DNT) decode_out_kernel(const __grid_constant__ DecodeArgs a, int b0, int nb) {
  using R = RowDot<Tc, float>;
  extern __shared__ __align__(16) float os[];  // [nb][Lq]
  const int n = blockIdx.x * (DNT / 32) + (threadIdx.x >> 5);
  const Tc* w = static_cast<const Tc*>(a.Wo) + (long long)n * a.Lq;
  uint4 first[R::NL];
  if (n < a.E) R::load(w, a.Lq, 0, first);
  pdl_wait();
  const float* o = a.o + (long long)b0 * a.Lq;
  for (int i = threadIdx.x * 4; i < nb * a.Lq; i += DNT * 4) cp_async16(os + i, o + i);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  if (n >= a.E) return;
  float acc[kGemvBatch];
#pragma unroll
  for (int b = 0; b < kGemvBatch; ++b) acc[b] = 0.f;
  R::run(w, a.Lq, os, nb, first, acc);
#pragma unroll
  for (int b = 0; b < kGemvBatch; ++b) {
    if (b < nb) {
      const float s = warp_sum(acc[b]);
      if ((threadIdx.x & 31) == 0) st_f(static_cast<To*>(a.y) + (long long)(b0 + b) * a.E + n, s);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// One head of the new token (es 2.B item 1): the causal seq conv (tap K-1 on this token, taps
// 0..K-2 on the conv state's rows, oldest first) and the head's d x d channel mix; the group's key
// head also makes the new v row (es 2.B item 3: channels [Lkv/2, Lkv) from the previous token).
// The conv state of the head's channels then advances by one token; each channel belongs to one
// CTA, so no other CTA reads what this one overwrites. The weights, the state rows and the previous
// v row are copied to shared memory before the wait for the down-projection.
template <typename Tc>
struct ConvSmem {
  // W_c rows padded by 16 bytes: the 16-byte pieces of eight consecutive rows at one column fall
  // in eight different bank groups
  __host__ __device__ static int wrow(int d) { return d + 16 / (int)sizeof(Tc); }
  // bytes: W_c [d][wrow] Tc, seq taps [d][K] Tc, state rows [K-1][d] Tc, previous v row [d] Tc,
  // then fp32 z [d] and seq-conv outputs [d]
  static size_t bytes(int d, int K) {
    const size_t e = sizeof(Tc);
    return (size_t)d * wrow(d) * e + (size_t)d * K * e + (size_t)(K - 1) * d * e + (size_t)d * e +
           2 * sizeof(float) * d;
  }
};

template <typename Tc>
__global__ void __launch_bounds__(DNT) decode_conv_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int V = Vec16<Tc>::N;
  pdl_launch_dependents();
  extern __shared__ __align__(16) unsigned char smc[];
  const int hh = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int d = a.d, K = a.K, wr = ConvSmem<Tc>::wrow(d);
  const bool isq = hh < a.G;
  const int L = isq ? a.Lq : a.Lkv;                  // width of this latent's state rows
  const int ch0 = isq ? (g * a.G + hh) * d : g * d;  // the head's first channel in q~ or k~
  Tc* wc_s = reinterpret_cast<Tc*>(smc);
  Tc* wseq_s = wc_s + d * wr;
  Tc* rows_s = wseq_s + d * K;
  Tc* vprev_s = rows_s + (K - 1) * d;
  float* z_s = reinterpret_cast<float*>(vprev_s + d);
  float* s_s = z_s + d;
  Tc* st = static_cast<Tc*>(a.conv_state) + (long long)b * ((long long)(K - 1) * (a.Lq + a.Lkv) + a.Lkv);
  Tc* rows = (isq ? st : st + (long long)(K - 1) * a.Lq) + ch0;  // row j of channel ch0 + i: rows[j*L + i]
  Tc* vrow = st + (long long)(K - 1) * (a.Lq + a.Lkv) + g * d;
  const Tc* wc = static_cast<const Tc*>(isq ? a.cq_chan : a.ck_chan) + (long long)(isq ? g * a.G + hh : g) * d * d;
  const Tc* wseq = static_cast<const Tc*>(isq ? a.cq_seq : a.ck_seq) + (long long)ch0 * K;
  for (int i = threadIdx.x * V; i < d * d; i += DNT * V) cp_async16(wc_s + (i / d) * wr + i % d, wc + i);
  for (int i = threadIdx.x * V; i < d * K; i += DNT * V) cp_async16(wseq_s + i, wseq + i);
  for (int i = threadIdx.x * V; i < (K - 1) * d; i += DNT * V) cp_async16(rows_s + i, rows + (long long)(i / d) * L + i % d);
  if (!isq)
    for (int i = threadIdx.x * V; i < d; i += DNT * V) cp_async16(vprev_s + i, vrow + i);
  cp_async_commit();
  pdl_wait();  // z from the down-projection
  const float* z = a.z + (long long)b * a.Nlat + (isq ? 0 : a.Lq) + ch0;
  const float* zv = a.z + (long long)b * a.Nlat + a.Lq + a.Lkv + g * d;
  float zvi = 0.f;
  for (int i = threadIdx.x; i < d; i += DNT) z_s[i] = z[i];
  if (!isq && threadIdx.x < d) zvi = zv[threadIdx.x];
  cp_async_wait<0>();
  __syncthreads();
  for (int i = threadIdx.x; i < d; i += DNT) {
    const float zi = z_s[i];
    const Tc* w = wseq_s + i * K;
    float acc = ld_f(w + K - 1) * zi;
    for (int j = 0; j < K - 1; ++j) acc = fmaf(ld_f(w + j), ld_f(rows_s + j * d + i), acc);
    s_s[i] = acc;
    for (int j = 0; j + 1 < K - 1; ++j) st_f(rows + (long long)j * L + i, ld_f(rows_s + (j + 1) * d + i));
    if (K > 1) st_f(rows + (long long)(K - 2) * L + i, zi);
  }
  if (!isq && threadIdx.x < d) {
    const int i = threadIdx.x;
    a.vt[(long long)b * a.Lkv + g * d + i] = (a.vshift && g * d + i >= a.vfrom) ? ld_f(vprev_s + i) : zvi;
    st_f(vrow + i, zvi);
  }
  __syncthreads();
  // out_i = sum_j W[i][j] s_j: tpr threads per row (lanes r and r + 32/tpr, ... of a warp), each
  // over d/tpr columns in 16-byte pieces
  float* out = a.c + (long long)b * (a.Lq + a.Lkv) + (isq ? 0 : a.Lq) + ch0;
  const int tpr = DNT / d < d / V ? DNT / d : d / V;  // threads per row: 2, 4 or 8
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rpw = 32 / tpr;
  const int row = warp * rpw + lane % rpw, part = lane / rpw;
  if (warp * rpw >= d) return;  // whole warps without a row
  const int cols = d / tpr;
  const Tc* wrp = wc_s + row * wr + part * cols;
  const float* sp = s_s + part * cols;
  float acc = 0.f;
  for (int c = 0; c < cols; c += V) {
    float wv[V];
    Vec16<Tc>::unpack(*reinterpret_cast<const uint4*>(wrp + c), wv);
#pragma unroll
    for (int k = 0; k < V; ++k) acc = fmaf(wv[k], sp[c + k], acc);
  }
  for (int off = rpw; off < 32; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (part == 0) out[row] = acc;
}

// ---------------------------------------------------------------------------------------------
// Attention of the new token over cache rows 0..t (es 2.A, 2.C: softmax attention on the compressed
// heads; the G query heads of a group share its K and V, so one pass over a key row serves all G).
template <typename Tc, int D, int GM>
struct AttnCfg {
  static constexpr int V = Vec16<Tc>::N;      // cache elements per 16-byte piece
  static constexpr int LPK = D / V;           // lanes per key row
  static constexpr int NKG = ANT / LPK;       // lane groups
  static constexpr int KB = GM <= 2 ? 8 : 4;  // keys per lane group per stage
  static constexpr int SK = KB * NKG;         // keys per stage
  static constexpr int STAGE = SK * 2 * D;    // Tc elements per stage: each key's K row, then its V row
  static constexpr int NS = (128 * 1024) / (STAGE * (int)sizeof(Tc));  // stages in a 128 KB ring
  static constexpr int PIECES = SK * 2 * LPK / ANT;  // 16-byte pieces per thread per stage
  static_assert(LPK >= 1 && LPK <= 32 && (LPK & (LPK - 1)) == 0, "lanes per key must divide a warp");
  static_assert(SK * 2 * LPK % ANT == 0 && NS >= 2, "stage shape");
  // shared memory (bytes): the ring, whose head holds the lane groups' partial outputs after the
  // body; the group's latents for the prologue; query rows; the new key and value rows; merge scratch
  static constexpr size_t RING = (size_t)NS * STAGE * sizeof(Tc);
  static_assert((size_t)NKG * GM * D * sizeof(float) <= RING, "partial outputs fit the ring");
  static constexpr size_t OFF_LAT = RING;  // zq [GM][D], zk [D], cq [GM][D], ck [D], v [D] (fp32)
  static constexpr size_t OFF_Q = OFF_LAT + sizeof(float) * (2 * GM + 3) * D;
  static constexpr size_t OFF_KV = OFF_Q + sizeof(float) * GM * D;
  static constexpr size_t OFF_SUB = OFF_KV + sizeof(float) * 2 * D;  // [ANT] float4 sums, [ANT] (max, sum)
  static constexpr size_t OFF_M = OFF_SUB + 24 * ANT;
  static constexpr size_t OFF_L = OFF_M + sizeof(float) * NKG * GM;
  static constexpr size_t OFF_FLAG = OFF_L + sizeof(float) * NKG * GM;
  static constexpr size_t SMEM = OFF_FLAG + 16;
};

template <typename Tc, int D, int GM>
__global__ void __launch_bounds__(ANT) decode_attn_kernel(const __grid_constant__ DecodeArgs a) {
  using C = AttnCfg<Tc, D, GM>;
  constexpr int V = C::V, LPK = C::LPK, NKG = C::NKG, KB = C::KB, SK = C::SK, NS = C::NS;
  pdl_launch_dependents();
  extern __shared__ __align__(16) unsigned char sma[];
  Tc* ring = reinterpret_cast<Tc*>(sma);
  float* lat = reinterpret_cast<float*>(sma + C::OFF_LAT);
  float* qf = reinterpret_cast<float*>(sma + C::OFF_Q);
  float* kv = reinterpret_cast<float*>(sma + C::OFF_KV);
  float* red_o = reinterpret_cast<float*>(sma);
  float4* sub = reinterpret_cast<float4*>(sma + C::OFF_SUB);
  float2* sub_ml = reinterpret_cast<float2*>(sma + C::OFF_SUB + 16 * ANT);
  float* red_m = reinterpret_cast<float*>(sma + C::OFF_M);
  float* red_l = reinterpret_cast<float*>(sma + C::OFF_L);
  int* flag = reinterpret_cast<int*>(sma + C::OFF_FLAG);
  const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = a.G, t = a.t, half = D / 2;
  const int k0 = chunk * a.chunk_len;
  const int k1 = min(k0 + a.chunk_len, t + 1);
  const int nst = (k1 - k0 + SK - 1) / SK;
  const long long rs = (long long)a.nkv * D;                           // cache row stride
  const long long cb = (long long)b * a.rows * rs + (long long)g * D;  // (sequence b, row 0, group g)
  const Tc* kcache = static_cast<const Tc*>(a.k_cache) + cb;
  const Tc* vcache = static_cast<const Tc*>(a.v_cache) + cb;

  // Stage s holds keys k0 + s*SK + r (r < SK). Rows before t are copied asynchronously (written by
  // earlier calls); row t, written by this step, comes from `kv` once the prologue has made it;
  // rows at or beyond k1 are zero.
  auto issue = [&](int s, bool row_t_ready) {
    if (s >= nst) return;
    Tc* slot = ring + (s % NS) * C::STAGE;
    const int kbase = k0 + s * SK;
#pragma unroll
    for (int i = 0; i < C::PIECES; ++i) {
      const int pi = threadIdx.x + i * ANT;
      const int r = pi / (2 * LPK), part = pi % (2 * LPK);
      const bool isv = part >= LPK;
      const int col = (part % LPK) * V;
      const int key = kbase + r;
      Tc* dst = slot + r * 2 * D + (isv ? D : 0) + col;
      if (key < t) {
        cp_async16(dst, (isv ? vcache : kcache) + key * rs + col);
      } else if (key == t) {
        if (row_t_ready) *reinterpret_cast<uint4*>(dst) = pack16(kv + (isv ? D : 0) + col, static_cast<Tc*>(nullptr));
      } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  };
#pragma unroll 1
  for (int s = 0; s < NS; ++s) {
    issue(s, false);
    cp_async_commit();
  }
  pdl_wait();  // z from the down-projection, c and the v row from the conv kernel

  // prologue: the group's latents in one round of copies, then QK-mean terms (es 2.B item 2) and
  // RoPE at position t of its query rows and key
  {
    const float* zb = a.z + (long long)b * a.Nlat;
    const float* cb_ = a.c + (long long)b * (a.Lq + a.Lkv);
    const float* src[5] = {zb + g * G * D, zb + a.Lq + g * D, a.K ? cb_ + g * G * D : nullptr,
                           a.K ? cb_ + a.Lq + g * D : nullptr,
                           a.K ? a.vt + (long long)b * a.Lkv + g * D : zb + a.Lq + a.Lkv + g * D};
    const int len[5] = {G * D, D, a.K ? G * D : 0, a.K ? D : 0, D};
    const int off[5] = {0, GM * D, (GM + 1) * D, (2 * GM + 1) * D, (2 * GM + 2) * D};
#pragma unroll
    for (int k = 0; k < 5; ++k)
      for (int i = threadIdx.x * 4; i < len[k]; i += ANT * 4) cp_async16(lat + off[k] + i, src[k] + i);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();
  {
    const float* zq = lat;
    const float* zk = lat + GM * D;
    const float* cq = a.K ? lat + (GM + 1) * D : zq;
    const float* ck = a.K ? lat + (2 * GM + 1) * D : zk;
    for (int e = threadIdx.x; e < (G + 1) * half; e += ANT) {
      const int hh = e / half, i = e % half;
      float v2[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int x = i + u * half;
        float val;
        if (hh < G) {
          val = cq[hh * D + x];
          if (a.mode & 1) val += 0.5f * (zq[hh * D + x] + zk[x]);
          if (a.mode & 2) val += 0.5f * (cq[hh * D + x] + ck[x]);
        } else {
          float mz = 0.f, mc = 0.f;
          for (int h = 0; h < G; ++h) {
            mz += zq[h * D + x];
            mc += cq[h * D + x];
          }
          val = ck[x];
          if (a.mode & 1) val += 0.5f * (mz / (float)G + zk[x]);
          if (a.mode & 2) val += 0.5f * (mc / (float)G + ck[x]);
        }
        v2[u] = val;
      }
      float* dst = hh < G ? qf + hh * D : kv;
      if (a.use_rope) {
        const float2 r = a.rot[i];
        dst[i] = v2[0] * r.x - v2[1] * r.y;
        dst[i + half] = v2[1] * r.x + v2[0] * r.y;
      } else {
        dst[i] = v2[0];
        dst[i + half] = v2[1];
      }
    }
    for (int i = threadIdx.x; i < D; i += ANT) kv[D + i] = lat[(2 * GM + 2) * D + i];
  }
  __syncthreads();
  if (t >= k0 && t < k1) {  // this chunk holds the new token: its cache row, and its ring slot if issued
    Tc* kc = static_cast<Tc*>(a.k_cache) + cb + t * rs;
    Tc* vc = static_cast<Tc*>(a.v_cache) + cb + t * rs;
    for (int i = threadIdx.x; i < D; i += ANT) {
      st_f(kc + i, kv[i]);
      st_f(vc + i, kv[D + i]);
    }
    const int st_ = (t - k0) / SK;
    if (st_ < NS && threadIdx.x < 2 * LPK) {
      const bool isv = threadIdx.x >= LPK;
      const int col = (threadIdx.x % LPK) * V;
      Tc* dst = ring + st_ * C::STAGE + ((t - k0) % SK) * 2 * D + (isv ? D : 0) + col;
      *reinterpret_cast<uint4*>(dst) = pack16(kv + (isv ? D : 0) + col, static_cast<Tc*>(nullptr));
    }
  }

  // body: lane group kg takes keys r = j*NKG + kg of each stage; lane p holds elements
  // [p*V, p*V + V) of q and o
  const int kg = threadIdx.x / LPK, p = threadIdx.x % LPK;
  float q[GM][V], o[GM][V], m[GM], l[GM];
#pragma unroll
  for (int h = 0; h < GM; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < V; ++e) {
      q[h][e] = h < G ? qf[h * D + p * V + e] * a.qscale : 0.f;
      o[h][e] = 0.f;
    }
  }
#pragma unroll 1
  for (int s = 0; s < nst; ++s) {
    cp_async_wait<NS - 1>();
    __syncthreads();
    const Tc* slot = ring + (s % NS) * C::STAGE;
    const int kbase = k0 + s * SK;
    float sc[KB][GM];
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      float kx[V];
      Vec16<Tc>::unpack(*reinterpret_cast<const uint4*>(slot + (j * NKG + kg) * 2 * D + p * V), kx);
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < V; ++e) acc = fmaf(q[h][e], kx[e], acc);
        sc[j][h] = acc;
      }
    }
#pragma unroll
    for (int off = LPK / 2; off > 0; off >>= 1)
#pragma unroll
      for (int j = 0; j < KB; ++j)
#pragma unroll
        for (int h = 0; h < GM; ++h) sc[j][h] += __shfl_xor_sync(0xffffffffu, sc[j][h], off);
    // online softmax per head (base 2): the scores become probabilities in place
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < KB; ++j)
        if (kbase + j * NKG + kg < k1) mx = fmaxf(mx, sc[j][h]);
      const float mnew = fmaxf(m[h], mx);
      const bool any = mnew != -INFINITY;
      const float corr = any ? exp2f(m[h] - mnew) : 1.f;
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < KB; ++j) {
        sc[j][h] = (any && kbase + j * NKG + kg < k1) ? exp2f(sc[j][h] - mnew) : 0.f;
        sum += sc[j][h];
      }
      l[h] = fmaf(l[h], corr, sum);
      m[h] = mnew;
#pragma unroll
      for (int e = 0; e < V; ++e) o[h][e] *= corr;
    }
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      float vx[V];
      Vec16<Tc>::unpack(*reinterpret_cast<const uint4*>(slot + (j * NKG + kg) * 2 * D + D + p * V), vx);
#pragma unroll
      for (int h = 0; h < GM; ++h)
#pragma unroll
        for (int e = 0; e < V; ++e) o[h][e] = fmaf(sc[j][h], vx[e], o[h][e]);
    }
    __syncthreads();  // the slot is free again
    issue(s + NS, true);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();

  // the CTA's lane groups merge into this chunk's partial result (output relative to its max)
  if (p == 0) {
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      red_m[kg * GM + h] = m[h];
      red_l[kg * GM + h] = l[h];
    }
  }
#pragma unroll
  for (int h = 0; h < GM; ++h)
#pragma unroll
    for (int e = 0; e < V; e += 4)
      *reinterpret_cast<float4*>(red_o + (kg * GM + h) * D + p * V + e) =
          make_float4(o[h][e], o[h][e + 1], o[h][e + 2], o[h][e + 3]);
  __syncthreads();
  const long long bg = (long long)b * a.nkv + g;
  float* po = a.part_o + (bg * a.nch + chunk) * G * D;
  float* pml = a.part_ml + (bg * a.nch + chunk) * G * 2;
  for (int idx = threadIdx.x; idx < G * D; idx += ANT) {
    const int h = idx / D, x = idx % D;
    float M = -INFINITY;
#pragma unroll 4
    for (int k = 0; k < NKG; ++k) M = fmaxf(M, red_m[k * GM + h]);
    float O = 0.f, Ls = 0.f;
#pragma unroll 4
    for (int k = 0; k < NKG; ++k) {
      const float mk = red_m[k * GM + h];
      const float w = mk == -INFINITY ? 0.f : exp2f(mk - M);
      O = fmaf(w, red_o[(k * GM + h) * D + x], O);
      Ls = fmaf(w, red_l[k * GM + h], Ls);
    }
    po[idx] = O;
    if (x == 0) {
      pml[2 * h] = M;
      pml[2 * h + 1] = Ls;
    }
  }
  // publish: every thread fences its own partial-row stores at device scope before the barrier, so
  // all of the CTA's stores are visible before thread 0's count can be seen (a fence by thread 0
  // alone orders only thread 0's stores: the last chunk could read other threads' rows before they
  // landed); the last chunk merges
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    *flag = atomicAdd(a.cnt + bg, 1);
    __threadfence();
  }
  __syncthreads();
  if (*flag != a.nch - 1) return;

  // the last chunk to finish merges the chunks of this (group, sequence): o = sum_c 2^(m_c - M) o_c /
  // sum_c 2^(m_c - M) l_c, in two rounds of loads: first every chunk's (max, sum) (thread c) and
  // from them the maxima M and the sums L per head; then thread (head, columns) reads its columns
  // of every chunk, a batch of independent loads at a time.
  {
    constexpr int NW = ANT / 32;
    constexpr int OPT = GM * D / ANT > 0 ? GM * D / ANT : 1;  // output columns per thread
    static_assert(OPT == 1 || OPT == 2 || OPT == 4, "output columns per thread");
    static_assert((size_t)kMaxChunks * GM * sizeof(float) <= C::RING, "merge weights fit the ring");
    static_assert(2 * GM * NW * sizeof(float) <= 24 * ANT, "merge sums fit the scratch");
    const float* po_all = a.part_o + bg * a.nch * G * D;
    const float* pml_all = a.part_ml + bg * a.nch * G * 2;
    float* wgt = reinterpret_cast<float*>(sma);                 // [nch][GM] weights, over the ring
    float* mred = reinterpret_cast<float*>(sma + C::OFF_SUB);  // [2][GM][NW] per-warp max and sum
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = threadIdx.x;  // nch <= kMaxChunks = ANT
    float cm[GM], cl[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      const float2 ml = (c < a.nch && h < G) ? __ldcg(reinterpret_cast<const float2*>(pml_all + (c * G + h) * 2))
                                             : make_float2(-INFINITY, 0.f);
      cm[h] = ml.x;
      cl[h] = ml.y;
      const float wm = warp_max(cm[h]);
      if (lane == 0) mred[h * NW + warp] = wm;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, mred[h * NW + w]);
      const float wc = cm[h] == -INFINITY ? 0.f : exp2f(cm[h] - M);
      if (c < a.nch) wgt[c * GM + h] = wc;
      const float ws = warp_sum(wc * cl[h]);
      if (lane == 0) mred[GM * NW + h * NW + warp] = ws;
    }
    __syncthreads();
    const int oh = threadIdx.x * OPT / D, oc = threadIdx.x * OPT % D;
    if (oh < G) {
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) L += mred[GM * NW + oh * NW + w];
      float r[OPT];
#pragma unroll
      for (int e = 0; e < OPT; ++e) r[e] = 0.f;
      constexpr int MB = 32;  // chunk values in flight per thread
      for (int c0 = 0; c0 < a.nch; c0 += MB) {
        float x[MB][OPT];
#pragma unroll
        for (int k = 0; k < MB; ++k) {
          const float* src = po_all + (long long)(c0 + k) * G * D + oh * D + oc;
#pragma unroll
          for (int e = 0; e < OPT; ++e) x[k][e] = c0 + k < a.nch ? __ldcg(src + e) : 0.f;
        }
        float ru[4][OPT];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int e = 0; e < OPT; ++e) ru[u][e] = 0.f;
#pragma unroll
        for (int k = 0; k < MB; ++k) {
          const float w = c0 + k < a.nch ? wgt[(c0 + k) * GM + oh] : 0.f;
#pragma unroll
          for (int e = 0; e < OPT; ++e) ru[k & 3][e] = fmaf(w, x[k][e], ru[k & 3][e]);
        }
#pragma unroll
        for (int e = 0; e < OPT; ++e) r[e] += (ru[0][e] + ru[1][e]) + (ru[2][e] + ru[3][e]);
      }
      const float li = 1.f / L;
#pragma unroll
      for (int e = 0; e < OPT; ++e) a.o[(long long)b * a.Lq + (long long)(g * G + oh) * D + oc + e] = r[e] * li;
    }
  }
}

// ---------------------------------------------------------------------------------------------
constexpr int kTargetCtas = 148;  // attention CTAs per step: one per SM of a B200

// Launch with programmatic stream serialization when `pdl`: the kernel may start once the previous
// kernel in the stream lets it, and waits for that kernel's completion itself (pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, size_t smem, cudaStream_t stream, bool pdl,
                     Args... args) {
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(DNT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Every kernel of the step is launched plainly: each starts once the one before it has completed.
// With programmatic dependent launch on the attention kernel, the two-step decode of two sequences
// produced a non-finite row in about one run in twenty; reading the chain did not show how, so no
// kernel of the step relies on early launch (the griddepcontrol instructions in the kernels are
// no-ops for a plain launch).
constexpr bool kDecodePdl = false;

template <typename Tc, int D>
cudaError_t launch_attn_g(const DecodeArgs& a, cudaStream_t stream) {
  static_assert(ANT == DNT, "one block size");
  const dim3 grid(a.nch, a.nkv, a.B);
  const bool pdl = kDecodePdl && a.K > 0;
  if (a.G <= 1) return launch_k(decode_attn_kernel<Tc, D, 1>, grid, AttnCfg<Tc, D, 1>::SMEM, stream, pdl, a);
  if (a.G <= 2) return launch_k(decode_attn_kernel<Tc, D, 2>, grid, AttnCfg<Tc, D, 2>::SMEM, stream, pdl, a);
  if (a.G <= 4) return launch_k(decode_attn_kernel<Tc, D, 4>, grid, AttnCfg<Tc, D, 4>::SMEM, stream, pdl, a);
  return launch_k(decode_attn_kernel<Tc, D, 8>, grid, AttnCfg<Tc, D, 8>::SMEM, stream, pdl, a);
}

template <typename Tc, typename To>
cudaError_t launch_typed(const DecodeArgs& a, cudaStream_t stream) {
  cudaError_t e;
  // 1. down-projection, kGemvBatch sequences per launch; the first launch of a step waits for
  //    everything before it in the stream
  for (int b0 = 0; b0 < a.B; b0 += kGemvBatch) {
    const int nb = a.B - b0 < kGemvBatch ? a.B - b0 : kGemvBatch;
    if ((e = launch_k(decode_down_kernel<Tc>, dim3((a.Nlat + DNT / 32 - 1) / (DNT / 32)),
                      sizeof(Tc) * (size_t)nb * a.E, stream, false, a, b0, nb)) != cudaSuccess)
      return e;
  }
  // 2. seq conv, channel mix, value shift, conv state
  if (a.K > 0 && (e = launch_k(decode_conv_kernel<Tc>, dim3(a.G + 1, a.nkv, a.B), ConvSmem<Tc>::bytes(a.d, a.K),
                               stream, kDecodePdl, a)) != cudaSuccess)
    return e;
  // 3. attention
  switch (a.d) {
    case 32: e = launch_attn_g<Tc, 32>(a, stream); break;
    case 64: e = launch_attn_g<Tc, 64>(a, stream); break;
    default: e = launch_attn_g<Tc, 128>(a, stream); break;
  }
  if (e != cudaSuccess) return e;
  // 4. output projection
  for (int b0 = 0; b0 < a.B; b0 += kGemvBatch) {
    const int nb = a.B - b0 < kGemvBatch ? a.B - b0 : kGemvBatch;
    if ((e = launch_k(decode_out_kernel<Tc, To>, dim3((a.E + DNT / 32 - 1) / (DNT / 32)),
                      sizeof(float) * (size_t)nb * a.Lq, stream, kDecodePdl, a, b0, nb)) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

// chunks per (KV group, sequence): one wave of CTAs over the SMs, at most kMaxChunks
int max_chunks(const BlockDims& dm) {
  const long long per = (long long)kTargetCtas / ((long long)dm.B * dm.nkv);
  return per < 1 ? 1 : (per > kMaxChunks ? kMaxChunks : (int)per);
}

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

struct DecodeLayout {
  size_t z, c, vt, o, part_o, part_ml, cnt, total;
};

DecodeLayout decode_layout(const BlockDims& dm) {
  DecodeLayout L;
  const size_t f = sizeof(float), B = (size_t)dm.B;
  const size_t parts = B * dm.nkv * (size_t)max_chunks(dm) * dm.G;
  size_t off = 0;
  L.z = off;
  off = up256(off + f * B * dm.Nlat);
  L.c = off;
  off = up256(off + f * B * (dm.Lq + dm.Lkv));
  L.vt = off;
  off = up256(off + f * B * dm.Lkv);
  L.o = off;
  off = up256(off + f * B * dm.Lq);
  L.part_o = off;
  off = up256(off + f * parts * dm.d);
  L.part_ml = off;
  off = up256(off + f * parts * 2);
  L.cnt = off;
  off = up256(off + sizeof(int) * B * dm.nkv);
  L.total = off;
  return L;
}

}  // namespace

bool decode_supported(const BlockDims& dm) {
  const bool dims = dm.d == 32 || dm.d == 64 || dm.d == 128;
  return dims && dm.G <= 8 && dm.E % 8 == 0 && dm.Lq % 8 == 0 && dm.B <= 65535 &&
         (size_t)kGemvBatch * dm.E * dtype_bytes(dm.io) <= 160 * 1024 &&
         (size_t)kGemvBatch * dm.Lq * sizeof(float) <= 160 * 1024 &&
         (dm.K == 0 || (dm.io == DType::BF16 ? ConvSmem<__nv_bfloat16>::bytes(dm.d, dm.K)
                                             : ConvSmem<float>::bytes(dm.d, dm.K)) <= 200 * 1024);
}

size_t decode_workspace_bytes(const BlockDims& dm) { return decode_layout(dm).total; }

cudaError_t launch_decode(const BlockDims& dm, const DecodePtrs& p, int cache_rows, cudaStream_t stream) {
  if (!decode_supported(dm)) return cudaErrorInvalidValue;
  DecodeArgs a{};
  a.x = p.x;
  a.Wq = p.Wq;
  a.Wk = p.Wk;
  a.Wv = p.Wv;
  a.cq_seq = p.cq_seq;
  a.cq_chan = p.cq_chan;
  a.ck_seq = p.ck_seq;
  a.ck_chan = p.ck_chan;
  a.Wo = p.Wo;
  a.y = p.y;
  a.k_cache = p.k_cache;
  a.v_cache = p.v_cache;
  a.conv_state = p.conv_state;
  const DecodeLayout L = decode_layout(dm);
  char* ws = static_cast<char*>(p.workspace);
  a.z = reinterpret_cast<float*>(ws + L.z);
  a.c = reinterpret_cast<float*>(ws + L.c);
  a.vt = reinterpret_cast<float*>(ws + L.vt);
  a.o = reinterpret_cast<float*>(ws + L.o);
  a.part_o = reinterpret_cast<float*>(ws + L.part_o);
  a.part_ml = reinterpret_cast<float*>(ws + L.part_ml);
  a.cnt = reinterpret_cast<int*>(ws + L.cnt);
  a.B = dm.B;
  a.E = dm.E;
  a.nkv = dm.nkv;
  a.d = dm.d;
  a.K = dm.K;
  a.G = dm.G;
  a.Lq = dm.Lq;
  a.Lkv = dm.Lkv;
  a.Nlat = dm.Nlat;
  a.t = dm.S - 1;
  a.rows = cache_rows;
  a.mode = dm.qk_mean_mode;
  a.vshift = dm.value_shift;
  a.vfrom = dm.vshift_from;
  a.use_rope = dm.use_rope;
  a.qscale = dm.scale * kLog2e;
  for (int i = 0; i < dm.d / 2; ++i) {
    const double ang = (double)a.t * pow((double)dm.rope_base, -2.0 * (double)i / (double)dm.d);
    a.rot[i] = make_float2((float)cos(ang), (float)sin(ang));
  }
  // key chunks of the t + 1 keys: as many as give every SM a CTA, each at least 64 keys
  const int n = a.t + 1, cmax = max_chunks(dm);
  int len = (n + cmax - 1) / cmax;
  if (len < 64) len = 64;
  a.chunk_len = len;
  a.nch = (n + len - 1) / len;
  if (dm.io == DType::BF16)
    return dm.out == DType::BF16 ? launch_typed<__nv_bfloat16, __nv_bfloat16>(a, stream)
                                 : launch_typed<__nv_bfloat16, float>(a, stream);
  return dm.out == DType::BF16 ? launch_typed<float, __nv_bfloat16>(a, stream) : launch_typed<float, float>(a, stream);
}

}  // namespace cca
