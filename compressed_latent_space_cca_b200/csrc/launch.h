// Internal launch interface between the C ABI (cca_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace cca {

// Element types that move between stages.
enum class DType : int { F32 = 0, BF16 = 1, F16 = 2 };

inline size_t dtype_bytes(DType t) { return t == DType::F32 ? 4 : 2; }

// Shape and options of one block, resolved from cca_config_t.
//
// Storage types: `io` is the type of the inputs and of the KV cache; `lat`
// the type of every intermediate (latents, attention q/k/v, attention
// output, the output-projection weight copy); `out` the type of y. For bf16
// blocks the intermediates are fp16: same tensor-core rate, 8x finer
// rounding, which keeps the chain of roundings inside the parity budget.
struct BlockDims {
  int B, S, E, nq, nkv, d, K;
  int G;        // nq / nkv
  int Lq, Lkv;  // nq*d, nkv*d
  int Nlat;     // Lq + 2*Lkv: width of the down-projection output
  long long T;  // B*S
  int qk_mean_mode, value_shift, use_rope;
  int vshift_from;  // V channels [vshift_from, Lkv) take the previous token (with value_shift)
  float rope_base, scale;
  DType io, lat, out;
};

// Pointers of one call (all device memory).
struct BlockPtrs {
  const void *x, *Wq, *Wk, *Wv, *cq_seq, *cq_chan, *ck_seq, *ck_chan, *Wo;
  void *y, *k_cache, *v_cache, *conv_state;
  // workspace
  void* qkv_lat;  // [T, Nlat] lat
  void* q;        // [T, Lq]  lat: attention queries
  void* k_att;    // [T, Lkv] lat: attention keys (== k_cache when lat == io)
  void* v_att;    // [T, Lkv] lat: attention values (== v_cache when lat == io)
  void* o;        // [T, Lq]  lat: attention output
  void* wo_lat;   // [E, Lq]  lat copy of W_o (== Wo when lat == io)
  void* wc_lat;   // [nq + nkv, d, d] lat copy of the channel-conv weights (null when lat == io)
  void* sched;    // scratch of the tensor-core attention (split-pair counters, partial rows)
  unsigned* dev_err;
  bool v_fused;   // the down-projection has written the V cache and v_att (value shift in its epilogue)
  // optional (non-null): the tensor-core attention also leaves the base-2 log-sum-exp of each row,
  // lse2[(b * nq + h) * lse_stride + t] = log2 sum_s 2^(scale log2(e) q_t . k_s)
  float* lse2;
  int lse_stride;
};

// ---- SIMT path (any dtype, any even head_dim <= 128) ----
// C[M, ldc] (cols [0,N)) = A[M,K] (row stride lda) * B[N,K]^T (row stride ldb)
cudaError_t launch_gemm_simt(DType in, DType out, const void* A, long long lda, const void* Bm, long long ldb,
                             void* C, long long ldc, long long M, int N, int K, cudaStream_t stream,
                             unsigned* dev_err);  // fp16 outputs beyond fp16's range are reported here
cudaError_t launch_attention_simt(const BlockDims& dm, const void* q, const void* k, const void* v, void* o,
                                  cudaStream_t stream);

// ---- preprocessing (seq conv, channel conv, QK-mean, RoPE, value shift) ----
cudaError_t launch_preproc_simt(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream);
cudaError_t launch_conv_state(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream);
// plain blocks (K == 0, no convolutions, QK-mean or value shift): RoPE on q and k, the KV cache
// and the attention copies, the W_o copy and the attention's split counters
cudaError_t launch_plain_preproc(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream);
// bf16 blocks with head_dim 128: channel mix on the tensor cores (mma.sync), coalesced I/O
bool preproc_tc_supported(const BlockDims& dm);
// The same steps as a persistent warp-specialised tcgen05 kernel (128-token tiles, every QK-mean and
// channel-mix term accumulated in tensor memory); needs the after-conv QK-mean and the fp16 W_c copy
// (wc_lat) scaled by kWsWeightScale.
constexpr float kWsWeightScale = 1.5f;
bool preproc_ws_supported(const BlockDims& dm);
cudaError_t launch_preproc_ws(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream);
cudaError_t launch_preproc_tc(const BlockDims& dm, const BlockPtrs& p, cudaStream_t stream);

// ---- tensor-core path (16-bit operands, sm_100a) ----
bool gemm_tc_supported(long long M, int N, int K);
// C[M, ldc] (cols [0,N)) = A[M,K] * [B0; B1; B2][N,K]^T, where the B operand
// is split by rows into up to three separate matrices. A and B share `in`
// (BF16 or F16); C is `out`.
struct GemmTcArgs {
  const void* A;
  long long M;
  int K;
  const void* B[3];
  int nrows[3];
  int nb;
  void* C;
  long long ldc;
  DType in, out;
  unsigned* dev_err;
  // optional side job of the epilogue warps before their first tile: side_dst[i][0, side_n[i]) =
  // fp16 copy of the bf16 side_src[i] times side_scale (0 means 1; fp16 overflow reported as a range
  // error)
  const void* side_src[2];
  void* side_dst[2];
  long long side_n[2];
  float side_scale;
  // optional value shift in the epilogue (non-null v_cache): output columns [v_col0, v_col0 + Lkv)
  // are v~ and go, shifted, to v_cache (bf16) and v_att (fp16) [T, Lkv] instead of C: channels
  // [vfrom, Lkv) move one row down within their sequence of S rows (zero at a sequence start) when
  // vshift is set
  void* v_cache;
  void* v_att;
  int v_col0, Lkv, S, vshift, vfrom;
  // optional split of K into ksplit slices (fp32 C only): each slice's product is added to C, which
  // the caller clears first
  int ksplit;
  // optional: A (B) holds only a_kwrap (b_kwrap) columns of K and repeats along it, column k of the
  // product reading its column k % a_kwrap (a multiple of 64, at most K; 0: A holds all K)
  int a_kwrap, b_kwrap;
  // optional: A stored [K][M] (row stride lda elements, 0: M) instead of [M][K]; B stored [K][N]
  // (row stride ldb, 0: N; one B matrix) instead of [N][K]. lda also sets a K-major A's row stride.
  int a_mn, b_mn;
  long long lda, ldb;
  // optional: the K columns A (B) actually holds when fewer than its wrap period (or K); the rest of
  // each period reads as zeros
  int a_kext, b_kext;
};
cudaError_t launch_gemm_tc(const GemmTcArgs& a, cudaStream_t stream);
// K slices for a GEMM with fewer 256 x 256 output tiles than the device has CTA pairs (1 otherwise):
// the count whose items fill the rounds of pairs best, with slices of at least 256 along K
int gemm_tc_ksplit(long long M, int N, int K);
// dst[0, n) = fp16 copy of the bf16 src times scale (fp16 overflow reported as a range error)
cudaError_t launch_convert_f16(const void* src, void* dst, long long n, unsigned* dev_err, cudaStream_t stream,
                               float scale = 1.0f);

bool attention_tc_supported(const BlockDims& dm);
cudaError_t launch_attention_tc(const BlockDims& dm, const void* q, const void* k, const void* v, void* o,
                                void* scratch, unsigned* dev_err, cudaStream_t stream, float* lse2 = nullptr,
                                int lse_stride = 0);
// Attention backward on the tensor cores (head_dim 128, fp16 operands): dq written, dk and dv added
// to (fp32, [B, S, width], scale applied); lse2 and delta [B][nq][stat_stride] (stat_stride a
// multiple of 64, >= S).
struct AttnBwdPtrs {
  const void *q, *k, *v, *dO;  // fp16, the forward's attention inputs and dL/dO
  const float *lse2, *delta;
  int stat_stride;
  float *dq, *dk, *dv;
};
bool attention_bwd_tc_supported(const BlockDims& dm);
cudaError_t launch_attention_bwd_tc(const BlockDims& dm, const AttnBwdPtrs& a, unsigned* dev_err,
                                    cudaStream_t stream);
// Split-pair scratch of the tensor-core attention: kAttnSplitCounters ints that must be zero when
// it starts (the preprocessing kernels clear them), then the partial rows.
constexpr int kAttnMaxSplit = 64;
constexpr int kAttnSplitCounters = kAttnMaxSplit * 2 * 8;
size_t attention_tc_scratch_bytes(const BlockDims& dm);

// ---- one decode step (token t = S - 1 of every sequence), fp32 arithmetic ----
struct DecodePtrs {
  const void *x, *Wq, *Wk, *Wv, *cq_seq, *cq_chan, *ck_seq, *ck_chan, *Wo;  // x: [B, E]
  void *y;                  // [B, E] out
  void *k_cache, *v_cache;  // [B, cache_rows, nkv, d]: rows 0..t-1 read, row t written
  void* conv_state;         // [B, (K-1)*(Lq+Lkv) + Lkv], advanced in place (NULL when K == 0)
  void* workspace;          // decode_workspace_bytes(dm), 256-byte aligned
};
// head_dim 32, 64 or 128; G <= 8; E and Lq multiples of 8
bool decode_supported(const BlockDims& dm);
size_t decode_workspace_bytes(const BlockDims& dm);  // independent of S
cudaError_t launch_decode(const BlockDims& dm, const DecodePtrs& p, int cache_rows, cudaStream_t stream);

// ---- backward of the block (fp32 arithmetic) ----
// dL/d(input) for the gradient dy of y, from the forward's activations (BlockPtrs, recomputed by
// the forward kernels). Every gradient is fp32 in its input's layout; dy is in `out`.
struct BackwardPtrs {
  const void* dy;  // [T, E]
  float *dx, *dWq, *dWk, *dWv, *dconvq_seq, *dconvq_chan, *dconvk_seq, *dconvk_chan, *dWo;
};
// Byte offsets (from the workspace start) of the backward's own buffers after the forward's
// `forward_bytes`: the forward's y, k_cache, v_cache, then fp32 dO, its fp16 copy dO16, lse, delta,
// dq, dk, dv, dc (channel-mix output gradient), dpre (latents' direct QK-mean gradient), ds
// (seq-conv output gradient), s (recomputed seq-conv output) and dlat (latents' gradient).
struct BackwardLayout {
  size_t y, k_cache, v_cache, dO, dO16, lse, delta, dq, dk, dv, dc, dpre, ds, s, dlat;
  // bf16 operands of the tensor-core GEMMs (token dimension padded to Tp in the transposed copies)
  size_t dy16, dy_t, x_t, o_t, dlat16, dlat_t, wo_t, w_t;
  size_t dw_all;  // fp32 [Nlat, E] scratch for the down-projection's weight gradients
  size_t total;
  int stat_stride;  // lse / delta rows of the tensor-core path: [B][nq][stat_stride]
  int Tp;           // tokens rounded up to a multiple of 64
};
// The channel-mix backward on the tensor cores (head_dim 128, K <= 8): ds written, dW_c added to
// (fp32; cleared by the caller)
bool chanmix_bwd_tc_supported(const BlockDims& dm);
cudaError_t launch_chanmix_bwd_tc(const BlockDims& dm, const float* dc, const void* lat, const void* cq_chan,
                                  const void* ck_chan, const void* cq_seq, const void* ck_seq, float* ds, float* dwq,
                                  float* dwk, unsigned* err, cudaStream_t stream);
// conv_kernel 0..8, head_dim <= 128 (even), io bf16 or fp32
bool backward_supported(const BlockDims& dm);
BackwardLayout backward_layout(const BlockDims& dm, size_t forward_bytes);
// tc_attention: the forward ran the tensor-core attention with p.lse2 set (BackwardLayout::lse);
// tc_gemm: the projections' shapes suit the tensor-core GEMM (bf16 blocks on sm_100)
cudaError_t launch_backward(const BlockDims& dm, const BlockPtrs& p, const BackwardPtrs& g, const BackwardLayout& L,
                            char* ws, cudaStream_t stream, bool tc_attention, bool tc_gemm);

// ---- misc ----
cudaError_t launch_wait_timeout_selftest(unsigned* dev_err, unsigned long long limit_ns, cudaStream_t stream);

// cuTensorMapEncodeTiled from the driver, fetched once through the runtime.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

int num_sms();

// Records msg as the calling thread's cca_last_error_message and returns status (an int
// holding a cca_status_t, so this header needs no C-ABI types).
int set_last_error(int status, const char* msg);

}  // namespace cca
