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
// its K/V head). The fp16 latents of all G+1 heads (32 tokens plus a K-1
// token halo) arrive in shared memory by cp.async, with the seq-conv taps of
// all G+1 heads. The heads' channel-mix weights (fp16 copies made once per
// call, exact for bf16 weights in fp16's normal range) stream in by cp.async
// through two buffers, so the next head's weights load while the current head
// is mixed. Per head the causal seq conv runs on
// CUDA cores in fp32 and its output s is rounded to fp16, so that the
// 32x128x128 channel mix runs on the tensor cores (mma.sync m16n8k16 fp16,
// fp32 accumulate): the rounding of s adds an error of the size of the fp16
// rounding that q and k get anyway. Each thread owns the same accumulator positions
// for every head, so c_k and the sum of the c_q stay in registers, and its
// columns come in pairs (c, c+64), so RoPE is applied in registers. Output
// tiles are staged in shared memory and written with 16-byte coalesced
// stores: q (fp16), the bf16 K cache and the fp16 attention copy of k; then
// the value shift copies v (bf16 cache and fp16 attention copy). Latent and s
// rows are padded to 272 bytes and weight rows are XOR-swizzled in 16-byte
// chunks, which keeps ldmatrix, the per-thread reads and the staging stores
// free of bank conflicts while two CTAs still fit on one SM.
#include <math.h>

#include "cca_common.cuh"
#include "launch.h"

namespace cca {
namespace {

constexpr int D = 128;
constexpr int TT = 32;          // tokens per CTA
constexpr int NT = 256;         // threads
constexpr int KMAX = 8;         // largest seq-conv kernel of this path
constexpr int GMAX = 8;         // largest group (query heads per KV head) of this path
constexpr int ROWH = D + 8;     // padded row, in 16-bit elements (272 bytes)
constexpr int WTILE = D * D;    // one head's channel weights, unpadded (swizzled) rows
constexpr int ZROWS = TT + KMAX - 1;
constexpr int KSTR = D + 4;     // padded fp32 row of the k stage

struct Theta {
  double v[D / 2];  // base^(-2i/d)
};

struct PreParams {
  const __half* lat;  // [T, Nlat] q~ | k~ | v~
  const __nv_bfloat16 *cq_seq, *ck_seq;
  const __half *cq_chan, *ck_chan;  // fp16 copies of the channel-conv weights
  __half* q;                          // [T, Lq]
  __nv_bfloat16 *k_cache, *v_cache;   // [T, Lkv]
  __half *k_att, *v_att;              // [T, Lkv]
  const __nv_bfloat16* wo;            // [E, Lq] (converted by a side job)
  __half* wo_lat;
  long long wo_n;
  unsigned* err;
  int* zero_cnt;  // split-pair counters of the attention launch that follows (cleared here)
  int S, nq, nkv, K, mode, vshift, vfrom, use_rope;
  int nbuf;  // weight buffers in shared memory: 2 (next head's weights prefetched) or 1
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0 source bytes: the 16 destination bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// wait until at most N of this thread's committed cp.async groups are pending
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

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

// Causal depthwise seq conv of one staged head into the bf16 hi / lo tiles. KC: the number of
// taps when known at compile time (0: p.K taps, at most KMAX). Row t of the output uses staged
// rows t .. t+K-1 (tap K-1 on the current token).
template <int KC>
__device__ __forceinline__ void seq_conv(const PreParams& p, const __half* zbuf, __half* sbuf,
                                         const __nv_bfloat16* wseq /* shared [D][K] */) {
  const int cp = threadIdx.x % (D / 2);  // column pair
  auto emit = [&](int t, float a0, float a1) {
    *reinterpret_cast<__half2*>(sbuf + t * ROWH + 2 * cp) = __floats2half2_rn(a0, a1);
  };
  auto zrow = [&](int r) { return __half22float2(*reinterpret_cast<const __half2*>(zbuf + r * ROWH + 2 * cp)); };
  if constexpr (KC > 0) {
    // each thread: one column pair, TPT consecutive tokens, the last KC latent rows in registers
    constexpr int TPT = TT / (NT / (D / 2));
    const int tb = (threadIdx.x / (D / 2)) * TPT;
    float2 w[KC], win[KC];
#pragma unroll
    for (int j = 0; j < KC; ++j)
      w[j] = make_float2(__bfloat162float(wseq[(2 * cp) * KC + j]), __bfloat162float(wseq[(2 * cp + 1) * KC + j]));
#pragma unroll
    for (int j = 0; j + 1 < KC; ++j) win[j] = zrow(tb + j);
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
      win[KC - 1] = zrow(tb + i + KC - 1);
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int j = 0; j < KC; ++j) fma2(a0, a1, w[j].x, w[j].y, win[j].x, win[j].y, a0, a1);
      emit(tb + i, a0, a1);
#pragma unroll
      for (int j = 0; j + 1 < KC; ++j) win[j] = win[j + 1];
    }
  } else {
    const int K = p.K;
    float w0[KMAX], w1[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      w0[j] = j < K ? __bfloat162float(wseq[(2 * cp) * K + j]) : 0.f;
      w1[j] = j < K ? __bfloat162float(wseq[(2 * cp + 1) * K + j]) : 0.f;
    }
    for (int t = threadIdx.x / (D / 2); t < TT; t += NT / (D / 2)) {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j < K) {
          const float2 z = zrow(t + j);
          a0 = fmaf(w0[j], z.x, a0);
          a1 = fmaf(w1[j], z.y, a1);
        }
      }
      emit(t, a0, a1);
    }
  }
}

// Channel mix of the warp's 16 rows x 4 n-tiles: acc[nt][0..3] (m16n8 layout), acc = s W^T
// (fp16 s and W, fp32 accumulation).
__device__ __forceinline__ void channel_mix(const __half* sbuf, const __half* wbuf, int rb, const int* ncol,
                                            float (&acc)[4][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  const int arow = (rb + (lane & 15)) * ROWH + (lane >> 4) * 8;
  const uint32_t abase = smem_u32(sbuf + arow);
  // B matrix m = lane / 8: rows ncol[0] + (m / 2) * 8 + (lane % 8), k chunk 2 ks + (m % 2), which
  // sits at chunk (2 ks) ^ y of the swizzled row, y = (m % 2) ^ (row % 8)
  const int brow = ncol[0] + ((lane >> 4) << 3) + (lane & 7);
  const int y = ((lane >> 3) & 1) ^ (lane & 7);
  const uint32_t brow0 = smem_u32(wbuf + brow * D);
  uint32_t bq[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) bq[j] = brow0 + (((2 * j) ^ y) << 4);
  constexpr uint32_t kB1 = 64 * D * 2;  // rows ncol[2] = ncol[0] + 64
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    uint32_t a0, a1, a2, a3, b0, b1, b2, b3, c0, c1, c2, c3;
    const uint32_t bk = bq[ks & 3] + (ks >> 2) * 128;
    ldsm_x4(abase + ks * 32, a0, a1, a2, a3);
    ldsm_x4(bk, b0, b1, b2, b3);
    ldsm_x4(bk + kB1, c0, c1, c2, c3);
    mma_f16_16816(acc[0], a0, a1, a2, a3, b0, b1);
    mma_f16_16816(acc[1], a0, a1, a2, a3, b2, b3);
    mma_f16_16816(acc[2], a0, a1, a2, a3, c0, c1);
    mma_f16_16816(acc[3], a0, a1, a2, a3, c2, c3);
  }
}

// Stream one head's channel-mix weights [out i][in j] (fp16) into wbuf: row i holds 16 chunks of
// 8 inputs, chunk c stored at position c ^ (i % 8).
__device__ __forceinline__ void load_weights_async(const __half* W, __half* wbuf) {
  // thread: chunk v of rows r, r + 16, ... (r % 8 and so the swizzle stay fixed)
  const int v = threadIdx.x % (D / 8), r = threadIdx.x / (D / 8);
  const uint32_t dst = smem_u32(wbuf + r * D + ((v ^ (r & 7)) << 3));
  const __half* src = W + r * D + v * 8;
  constexpr int kRows = NT / (D / 8);
#pragma unroll
  for (int k = 0; k < D / kRows; ++k) cp_async16(dst + k * kRows * D * 2, src + k * kRows * D, true);
}

// Byte offset of the RoPE tables: after the weight buffers, the s tile, the latents and the seq taps.
__host__ __device__ __forceinline__ size_t rope_table_offset(int H1, int K, int nbuf) {
  const size_t end = 2 * ((size_t)nbuf * WTILE + (size_t)TT * ROWH + (size_t)H1 * (TT + K - 1) * ROWH +
                          (size_t)H1 * D * K);
  return (end + 15) & ~(size_t)15;
}

// MINB: CTAs per SM the launch is built for (2, or 3 with one weight buffer and 80 registers)
template <int KC, int MINB>
__global__ void __launch_bounds__(NT, MINB) preproc_tc_kernel(const __grid_constant__ PreParams p,
                                                          const __grid_constant__ Theta th) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int G = p.nq / p.nkv;
  const int H1 = G + 1;
  const int KK = KC > 0 ? KC : p.K;  // seq-conv taps
  const int ZR = TT + KK - 1;        // staged rows per head
  __half* wbuf = reinterpret_cast<__half*>(smem_raw);  // nbuf x [D][D] channel weights (fp16)
  __half* sbuf = wbuf + p.nbuf * WTILE;                // [TT][ROWH] seq-conv output s (fp16)
  __half* zall = sbuf + TT * ROWH;                     // [H1][ZR][ROWH] latents; head G = k
  __nv_bfloat16* wsq = reinterpret_cast<__nv_bfloat16*>(zall + H1 * ZR * ROWH);  // [H1][D][K] seq taps
  float2* rtab = reinterpret_cast<float2*>(smem_raw + rope_table_offset(H1, KK, p.nbuf));  // [2][D/2] RoPE
  __half* stage = sbuf;                                               // [TT][ROWH] q output stage
  float* kst = reinterpret_cast<float*>(wbuf);                        // [TT][KSTR] k stage (fp32)
  // weights of the i-th head in processing order (0: the K head, then query heads 0..G-1)
  auto wslot = [&](int i) { return wbuf + (p.nbuf == 2 ? (i & 1) : 0) * WTILE; };

  const int Lq = p.nq * D, Lkv = p.nkv * D, Nlat = Lq + 2 * Lkv;
  const int t0 = blockIdx.x * TT, g = blockIdx.y, b = blockIdx.z;
  const long long rowbase = (long long)b * p.S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = (warp & 1) * 16;  // warp rows
  const int cg = warp >> 1;        // column group: cols [16cg, 16cg+16) and the same +64
  const int ncol[4] = {cg * 16, cg * 16 + 8, 64 + cg * 16, 64 + cg * 16 + 8};
  const int r0 = rb + (lane >> 2), r1 = r0 + 8;
  const int cq = (lane & 3) * 2;
  const int zr0 = r0 + KK - 1, zr1 = r1 + KK - 1;  // current-token rows in the latent tiles
  bool bad = false;
  float amax = 0.f;  // largest |q|, |k| of this thread

  // ---- all latents of the group (query heads 0..G-1, then the K head) and the K head's weights
  for (int R = threadIdx.x / (D / 8); R < H1 * ZR; R += NT / (D / 8)) {
    const int v = threadIdx.x % (D / 8), hh = R / ZR, r = R - hh * ZR;
    const int t = t0 - (KK - 1) + r;
    const int col = (hh < G) ? (g * G + hh) * D : Lq + g * D;
    const bool ok = t >= 0 && t < p.S;
    cp_async16(smem_u32(zall + (hh * ZR + r) * ROWH + v * 8), p.lat + (rowbase + (ok ? t : 0)) * Nlat + col + v * 8,
               ok);
  }
  load_weights_async(p.ck_chan + (long long)g * D * D, wslot(0));
  cp_async_commit();
  if (p.nbuf == 2) load_weights_async(p.cq_chan + (long long)g * G * D * D, wslot(1));
  cp_async_commit();  // (an empty group when nbuf == 1)
  // seq-conv taps of the group's heads, [H1][D][K]: query heads g*G .. g*G+G-1 (contiguous in
  // cq_seq), then the K head; 16-byte vectors when both sources allow them
  {
    const __nv_bfloat16* qs = p.cq_seq + (long long)g * G * D * KK;
    const __nv_bfloat16* ks = p.ck_seq + (long long)g * D * KK;
    if (((reinterpret_cast<uintptr_t>(qs) | reinterpret_cast<uintptr_t>(ks)) & 15) == 0) {
      const int nq8 = G * D * KK / 8, n8 = H1 * D * KK / 8;  // D * KK is a multiple of 8
      for (int v = threadIdx.x; v < n8; v += NT)
        reinterpret_cast<uint4*>(wsq)[v] =
            v < nq8 ? reinterpret_cast<const uint4*>(qs)[v] : reinterpret_cast<const uint4*>(ks)[v - nq8];
    } else {
      for (int e = threadIdx.x; e < H1 * D * KK; e += NT)
        wsq[e] = e < G * D * KK ? qs[e] : ks[e - G * D * KK];
    }
  }

  // ---- side job, issued while the copies are in flight: this CTA's slice of W_o as fp16 (8-element vectors)
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
    if (p.zero_cnt != nullptr && cid == 0)
      for (int i = threadIdx.x; i < kAttnSplitCounters; i += NT) p.zero_cnt[i] = 0;
  }

  // RoPE tables: rtab[i] = (cos, sin) of t0 * theta_i, rtab[D/2 + i] = (cos, sin) of 8 * theta_i
  if (p.use_rope && threadIdx.x < D) {
    const int i = threadIdx.x % (D / 2);
    float c, sn;
    if (threadIdx.x < D / 2) {
      const double a = (double)t0 * th.v[i];
      // reduce a modulo 2 pi with 2 pi split into a high and a low double
      const double k = rint(a * 0.15915494309189535);
      double r = fma(-k, 6.283185307179586, a);
      r = fma(-k, 2.4492935982947064e-16, r);
      sincosf((float)r, &sn, &c);
    } else {
      sincosf((float)(8.0 * th.v[i]), &sn, &c);  // at most 8 radians
    }
    rtab[threadIdx.x] = make_float2(c, sn);
  }
  float rc[2][4], rs[2][4];  // RoPE factors, filled once the tables are in shared memory
  auto rope = [&](float (&v)[4][4]) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x1 = v[nt][e], x2 = v[nt + 2][e];
        v[nt][e] = x1 * rc[nt][e] - x2 * rs[nt][e];
        v[nt + 2][e] = x2 * rc[nt][e] + x1 * rs[nt][e];
      }
  };
  // latents of head hh at this thread's two adjacent columns of n-tile nt, row r0 (rs = 0) or r1
  auto zpair = [&](int hh, int nt, int rs) -> float2 {
    return __half22float2(*reinterpret_cast<const __half2*>(zall + (hh * ZR + (rs ? zr1 : zr0)) * ROWH + ncol[nt] + cq));
  };

  // ---- the K head: conv + channel mix, c_k kept in registers
  cp_async_wait<1>();  // latents and the K head's weights
  __syncthreads();

  // RoPE factors of this thread's (row, column < 64) positions, [nt<2][e]: the angle of row r0 is
  // t0 theta + r0 theta (r0 theta < 24 radians, reduced in fp32), row r1 = r0 + 8 adds 8 theta
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e1 = 0; e1 < 2; ++e1) {
      const int i = ncol[nt] + cq + e1;
      float c0 = 1.f, s0 = 0.f, c1 = 1.f, s1 = 0.f;
      if (p.use_rope) {
        const float a = (float)((double)r0 * th.v[i]);
        const float k = rintf(a * 0.15915494f);
        float r = fmaf(-k, 6.28318548f, a);  // 2 pi = 6.28318548f - 1.7484555e-7f
        r = fmaf(k, 1.7484555e-7f, r);
        float ca, sa;
        __sincosf(r, &sa, &ca);
        const float2 b = rtab[i], d8 = rtab[D / 2 + i];
        c0 = b.x * ca - b.y * sa;
        s0 = b.y * ca + b.x * sa;
        c1 = c0 * d8.x - s0 * d8.y;
        s1 = s0 * d8.x + c0 * d8.y;
      }
      rc[nt][e1] = c0;
      rs[nt][e1] = s0;
      rc[nt][2 + e1] = c1;
      rs[nt][2 + e1] = s1;
    }
  seq_conv<KC>(p, zall + G * ZR * ROWH, sbuf, wsq + G * D * KK);
  __syncthreads();
  float ck[4][4];
  channel_mix(sbuf, wslot(0), rb, ncol, ck);
  float csum[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) csum[nt][e] = 0.f;

  // ---- the G query heads
  for (int hh = 0; hh < G; ++hh) {
    const int h = g * G + hh;
    __syncthreads();  // sbuf and the previous head's weight buffer are free
    // weights of query head hh + 1 (double buffering) or hh (single buffer)
    const int next = p.nbuf == 2 ? hh + 1 : hh;
    const bool issue = next < G;
    if (issue) load_weights_async(p.cq_chan + (long long)(g * G + next) * D * D, wslot(next + 1));
    cp_async_commit();
    seq_conv<KC>(p, zall + hh * ZR * ROWH, sbuf, wsq + hh * D * KK);
    if (p.nbuf == 2) cp_async_wait<1>();  // all but the group just committed: head hh's weights
    else cp_async_wait<0>();
    __syncthreads();
    float acc[4][4];
    channel_mix(sbuf, wslot(hh + 1), rb, ncol, acc);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int rs = 0; rs < 2; ++rs) {
        float2 pre = make_float2(0.f, 0.f);
        if (p.mode & 1) {
          const float2 zq = zpair(hh, nt, rs), zk = zpair(G, nt, rs);
          pre = make_float2(0.5f * (zq.x + zk.x), 0.5f * (zq.y + zk.y));
        }
#pragma unroll
        for (int e1 = 0; e1 < 2; ++e1) {
          const int e = 2 * rs + e1;
          float v = acc[nt][e] + (e1 ? pre.y : pre.x);
          if (p.mode & 2) v += 0.5f * (acc[nt][e] + ck[nt][e]);
          csum[nt][e] += acc[nt][e];
          acc[nt][e] = v;
        }
      }
    if (p.use_rope) rope(acc);
    __syncthreads();  // sbuf becomes the q stage
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int col = ncol[nt] + cq;
      *reinterpret_cast<__half2*>(stage + r0 * ROWH + col) = __floats2half2_rn(acc[nt][0], acc[nt][1]);
      *reinterpret_cast<__half2*>(stage + r1 * ROWH + col) = __floats2half2_rn(acc[nt][2], acc[nt][3]);
#pragma unroll
      for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(acc[nt][e]));
    }
    __syncthreads();
    for (int e = threadIdx.x; e < TT * (D / 8); e += NT) {
      const int r = e / (D / 8), v = e % (D / 8);
      if (t0 + r < p.S)
        *reinterpret_cast<uint4*>(p.q + (rowbase + t0 + r) * Lq + (long long)h * D + v * 8) =
            *reinterpret_cast<const uint4*>(stage + r * ROWH + v * 8);
    }
  }

  // value-shift sources, loaded now so that the latency overlaps the k combine: channels
  // [vfrom, Lkv) come from the previous token (8-channel vectors never straddle the boundary)
  static_assert(TT * (D / 8) == 2 * NT, "two value vectors per thread");
  uint4 vsrc[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int e = threadIdx.x + i * NT, r = e / (D / 8), v = e % (D / 8);
    const int t = t0 + r, gc = g * D + v * 8;
    const int src = (p.vshift && gc >= p.vfrom) ? t - 1 : t;
    vsrc[i] = make_uint4(0, 0, 0, 0);
    if (t < p.S && src >= 0) vsrc[i] = *reinterpret_cast<const uint4*>(p.lat + (rowbase + src) * Nlat + Lq + Lkv + gc);
  }

  // ---- k = c_k + means, RoPE; staged in fp32, written as the bf16 cache and the fp16 copy
  {
    const float invG = 1.f / (float)G;
    float val[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int rs = 0; rs < 2; ++rs) {
        float2 pre = make_float2(0.f, 0.f);
        if (p.mode & 1) {
          float2 mq = make_float2(0.f, 0.f);
          for (int hh = 0; hh < G; ++hh) {
            const float2 z = zpair(hh, nt, rs);
            mq.x += z.x;
            mq.y += z.y;
          }
          const float2 zk = zpair(G, nt, rs);
          pre = make_float2(0.5f * (mq.x * invG + zk.x), 0.5f * (mq.y * invG + zk.y));
        }
#pragma unroll
        for (int e1 = 0; e1 < 2; ++e1) {
          const int e = 2 * rs + e1;
          float v = ck[nt][e] + (e1 ? pre.y : pre.x);
          if (p.mode & 2) v += 0.5f * (csum[nt][e] * invG + ck[nt][e]);
          val[nt][e] = v;
        }
      }
    if (p.use_rope) rope(val);
    __syncthreads();  // wbuf becomes the k stage
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int col = ncol[nt] + cq;
      *reinterpret_cast<float2*>(kst + r0 * KSTR + col) = make_float2(val[nt][0], val[nt][1]);
      *reinterpret_cast<float2*>(kst + r1 * KSTR + col) = make_float2(val[nt][2], val[nt][3]);
#pragma unroll
      for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(val[nt][e]));
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < TT * (D / 8); e += NT) {
    const int r = e / (D / 8), v = e % (D / 8);
    if (t0 + r >= p.S) continue;
    const float4 lo = *reinterpret_cast<const float4*>(kst + r * KSTR + v * 8);
    const float4 hi = *reinterpret_cast<const float4*>(kst + r * KSTR + v * 8 + 4);
    const long long off = (rowbase + t0 + r) * Lkv + (long long)g * D + v * 8;
    *reinterpret_cast<uint4*>(p.k_cache + off) =
        make_uint4(pack_bf16x2(lo.x, lo.y), pack_bf16x2(lo.z, lo.w), pack_bf16x2(hi.x, hi.y), pack_bf16x2(hi.z, hi.w));
    *reinterpret_cast<uint4*>(p.k_att + off) =
        make_uint4(pack_f16x2(lo.x, lo.y), pack_f16x2(lo.z, lo.w), pack_f16x2(hi.x, hi.y), pack_f16x2(hi.z, hi.w));
  }

  // ---- value shift: the bf16 cache and the fp16 attention copy of the shifted v
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int e = threadIdx.x + i * NT, r = e / (D / 8), v = e % (D / 8);
    const int t = t0 + r, gc = g * D + v * 8;
    if (t >= p.S) continue;
    const uint4 hv = vsrc[i];
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

  // q and k leave as fp16: any of this thread's values beyond fp16's range (infinities included)
  report_range(bad || amax > 65504.0f, p.err);
}

size_t smem_bytes(int G, int K, int nbuf) { return rope_table_offset(G + 1, K, nbuf) + sizeof(float2) * D; }

// Occupancy of a shape (228 KB of shared memory per SM, 1 KB reserved per CTA): three CTAs per SM
// with one weight buffer when they fit (the warps of the other CTAs hide the unprefetched weights;
// 80 registers, a few spilled: measured 52.3 -> 50.1 us at S=16384, G=2), else two CTAs with two
// weight buffers (the next head's weights prefetched), else two or one with one buffer.
int ctas_per_sm(int G, int K) { return smem_bytes(G, K, 1) + 1024 <= 76 * 1024 ? 3 : 2; }
int weight_buffers(int G, int K) {
  return ctas_per_sm(G, K) == 3 || smem_bytes(G, K, 2) + 1024 > 114 * 1024 ? 1 : 2;
}

}  // namespace

bool preproc_tc_supported(const BlockDims& dm) {
  return dm.io == DType::BF16 && dm.lat == DType::F16 && dm.d == D && dm.K >= 1 && dm.K <= KMAX && dm.G <= GMAX &&
         ((long long)dm.E * dm.Lq) % 8 == 0;
}

cudaError_t launch_preproc_tc(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream) {
  if (!preproc_tc_supported(dm)) return cudaErrorInvalidValue;
  PreParams q;
  q.lat = static_cast<const __half*>(p.qkv_lat);
  q.cq_seq = static_cast<const __nv_bfloat16*>(p.cq_seq);
  q.cq_chan = static_cast<const __half*>(p.wc_lat);
  q.ck_seq = static_cast<const __nv_bfloat16*>(p.ck_seq);
  q.ck_chan = static_cast<const __half*>(p.wc_lat) + (long long)dm.nq * D * D;
  q.q = static_cast<__half*>(p.q);
  q.k_cache = static_cast<__nv_bfloat16*>(p.k_cache);
  q.v_cache = static_cast<__nv_bfloat16*>(p.v_cache);
  q.k_att = static_cast<__half*>(p.k_att);
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
  q.vfrom = dm.vshift_from;
  q.use_rope = dm.use_rope;
  Theta th;
  for (int i = 0; i < D / 2; ++i) th.v[i] = pow((double)dm.rope_base, -2.0 * (double)i / (double)D);
  q.nbuf = weight_buffers(dm.G, dm.K);
  const size_t smem = smem_bytes(dm.G, dm.K, q.nbuf);
  dim3 grid((dm.S + TT - 1) / TT, dm.nkv, dm.B);
  const bool three = ctas_per_sm(dm.G, dm.K) == 3;
  auto kern = dm.K == 4 ? (three ? preproc_tc_kernel<4, 3> : preproc_tc_kernel<4, 2>)
                        : (three ? preproc_tc_kernel<0, 3> : preproc_tc_kernel<0, 2>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, NT, smem, stream>>>(q, th);
  return cudaGetLastError();
}

}  // namespace cca
