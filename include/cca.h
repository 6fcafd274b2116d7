/*
 * cca.h - C ABI of the B200 prefill library for one Compressed Convolutional
 * Attention (CCA) / CCGQA block.
 *
 * The operation is the block described in "Compressed Convolutional
 * Attention: Efficient Attention in a Compressed Latent Space"
 * (gist.science/es/paper/2510.04476, section 2; French twin
 * gist.science/fr/paper/2510.04476, section 2):
 *
 *   q~, k~, v~ = x W_q^T, x W_k^T, x W_v^T        latent width E/C  (es 2.A)
 *   q, k       = causal seq conv -> per-head channel conv of q~, k~ (es 2.B.1)
 *                + QK-mean before and after the convs             (es 2.B.2)
 *                then RoPE in the latent                          (es 3, item 2)
 *   v          = value shift of v~: the upper half of the latent
 *                channels comes from the previous token           (es 2.B.3)
 *   o          = causal softmax(q k^T / sqrt(d)) v, K/V head g serves the
 *                query heads g*G .. g*G+G-1 (G = n_q / n_kv)      (es 2.A, 2.C)
 *   y          = o W_o^T                                           (implied)
 *
 * and the compressed KV cache (k after RoPE, v after the shift).
 *
 * Conventions for every call below:
 *   - Pointers named *_host are host memory; every other data pointer is
 *     device memory of the current CUDA device. The caller allocates and owns
 *     all of it. The library allocates nothing per call.
 *   - All tensors are dense and row-major (the last index is contiguous) and
 *     start on a 16-byte boundary. Element type is cfg->dtype unless noted.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and nothing synchronizes except cca_poll_device_status.
 *   - Invalid arguments are rejected before any launch; outputs are then left
 *     untouched. cca_last_error_message() gives a one-line reason.
 *   - Calls on distinct streams may run concurrently if they use distinct
 *     workspaces and outputs.
 */
#ifndef CCA_H_
#define CCA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CCA_VERSION 1

typedef enum cca_status {
  CCA_OK = 0,
  CCA_ERR_INVALID_ARG = 1,    /* a shape, pointer, mode or alignment is invalid */
  CCA_ERR_UNSUPPORTED = 2,    /* valid block, but no kernel for this shape/dtype */
  CCA_ERR_WORKSPACE = 3,      /* workspace missing or smaller than cca_workspace_size */
  CCA_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
  CCA_ERR_DEVICE_TIMEOUT = 5, /* a bounded device-side wait gave up (see cca_poll_device_status) */
  CCA_ERR_NUMERIC_RANGE = 6   /* an fp16 intermediate overflowed (see cca_poll_device_status) */
} cca_status_t;

typedef enum cca_dtype {
  CCA_F32 = 0,   /* float32 */
  CCA_BF16 = 1,  /* bfloat16 */
  CCA_F16 = 2    /* float16: only as the type of bf16 blocks' intermediates */
} cca_dtype_t;

/* QK-mean mode bits (es 2.B item 2: the mean of q and k taken before and
 * after the convolution is added to the conv outputs). */
#define CCA_QK_MEAN_PRE 1
#define CCA_QK_MEAN_POST 2

/* Block shape and options. Field order is part of the ABI. */
typedef struct cca_config {
  int batch;         /* B >= 1 independent sequences */
  int seq_len;       /* S >= 1 tokens per sequence */
  int hidden;        /* E */
  int C;             /* compression factor: hidden == C * n_q_heads * head_dim */
  int n_q_heads;     /* query heads in the latent */
  int n_kv_heads;    /* K/V heads; n_q_heads % n_kv_heads == 0 (CCGQA when <) */
  int head_dim;      /* d, even */
  int conv_kernel;   /* K >= 1 taps of the causal sequence conv; 0: a plain attention block
                        (no convolutions, the uncompressed baseline when C = 1): qk_mean_mode and
                        value_shift must be 0, the four conv weight pointers may be NULL and
                        conv_state must be NULL */
  int qk_mean_mode;  /* OR of CCA_QK_MEAN_*; 3 is the method as described */
  int value_shift;   /* 1 = shift the upper half of v's channels by one token */
  int use_rope;      /* 1 = rotate-half RoPE on q and k */
  float rope_base;   /* RoPE base, e.g. 10000 */
  float softmax_scale; /* 0 => 1/sqrt(head_dim) */
  int dtype;         /* cca_dtype_t of every input, the KV cache and the conv state */
  int out_dtype;     /* cca_dtype_t of y (CCA_F32 allowed for bf16 inputs) */
  /* A block that holds some of the KV groups of a wider block (heads split over GPUs: the QK-mean
   * couples a query head only with its own group, so each share of groups is a block of its own,
   * and y is the sum of the shares' outputs). The value shift divides the WHOLE block's V channels
   * in halves (es 2.B item 3), so a share needs to know where its channels sit:
   *   kv_channel_offset  the wider block's V channel index of this block's V channel 0 (a multiple
   *                      of 8; 0 for a whole block)
   *   kv_total_channels  the wider block's V width n_kv_total * head_dim (a multiple of 16, at
   *                      least kv_channel_offset + n_kv_heads * head_dim; 0 for a whole block)
   * This block's V channel c takes the previous token when value_shift is set and
   * kv_channel_offset + c >= kv_total_channels / 2. */
  int kv_channel_offset;
  int kv_total_channels;
} cca_config_t;

/* Kernel path selection (cca_prefill_ex). AUTO runs each stage on its
 * tensor-core kernel (tcgen05/TMEM fed by TMA, sm_100 only) when that kernel
 * takes the shape (bf16; head_dim 128 for attention and preprocessing) and on
 * its SIMT kernel otherwise; its preprocessing is the tcgen05 kernel when the
 * QK-mean includes the after-conv term (CCA_QK_MEAN_POST) and the mma.sync
 * kernel otherwise. SIMT forces every stage onto the SIMT kernels; TENSOR
 * requires the tensor-core kernels for every stage (preprocessing: mma.sync). */
typedef enum cca_path {
  CCA_PATH_AUTO = 0,
  CCA_PATH_SIMT = 1,
  CCA_PATH_TENSOR = 2   /* CCA_ERR_UNSUPPORTED if the shape does not allow it */
} cca_path_t;
/* Per-stage choice: bit0 down-projection, bit1 attention, bit2 output
 * projection, bit3 preprocessing on the tensor-core kernel (channel mix on
 * mma.sync), bit4 preprocessing on the tcgen05 kernel (channel mix as
 * tcgen05 MMAs into tensor memory; bits 3 and 4 exclude each other), bit5
 * (with bits 0 and 4) the value shift fused into the down-projection: its
 * epilogue writes the V cache and the attention copy of v directly, so the
 * V latent never makes the round trip through memory (the v~ region of the
 * workspace is then not written; with a conv_state the shift stays in the
 * preprocessing kernel, which needs the last v~ row); the other stages on
 * SIMT. */
#define CCA_PATH_TENSOR_MASK(bits) (0x100 | ((bits) & 63))

/* Which kernels a call would launch (cca_plan). */
typedef struct cca_plan {
  int down_proj_tensor;   /* 1: tcgen05 GEMM, 0: SIMT GEMM (three launches) */
  int attention_tensor;   /* 1: tcgen05 flash attention, 0: SIMT attention */
  int out_proj_tensor;    /* 1: tcgen05 GEMM, 0: SIMT GEMM */
  int preproc_tensor;     /* 1: preprocessing with the channel mix on mma.sync, 2: on tcgen05 */
  int launches;           /* kernel launches of one cca_prefill without conv_state */
  int value_shift_fused;  /* 1: the value shift runs in the down-projection's epilogue (path bit 5) */
} cca_plan_t;

typedef struct cca_prefill_opts {
  int path;              /* cca_path_t */
  /* If non-NULL: five cudaEvent_t recorded on `stream` before the down-
   * projection, before preprocessing, before attention, before the output
   * projection and after it. Owned by the caller. */
  void* const* stage_events;
} cca_prefill_opts_t;

/* Byte offsets of the intermediates inside the workspace, for inspection
 * after a call has completed. Each region is row-major of type lat_dtype,
 * T = batch * seq_len. Intermediates of fp32 blocks are fp32; those of bf16
 * blocks are fp16 (same tensor-core rate as bf16, 8x finer rounding), which
 * keeps the block's chain of roundings small; inputs, the KV cache and y keep
 * cfg->dtype / cfg->out_dtype. For fp32 blocks the k_att / v_att / W_o
 * regions are empty (the attention reads the KV cache and W_o directly), and
 * so is the W_c region. */
typedef struct cca_workspace_layout {
  size_t total_bytes;
  size_t elem_bytes;        /* bytes per intermediate element */
  int lat_dtype;            /* cca_dtype_t of the intermediates */
  int reserved;
  size_t qkv_lat_offset;    /* [T, Lq + 2*Lkv]: q~ | k~ | v~ (down-projection) */
  size_t q_offset;          /* [T, Lq]: q after convs, QK-mean and RoPE */
  size_t k_att_offset;      /* [T, Lkv]: k as the attention reads it */
  size_t v_att_offset;      /* [T, Lkv]: v as the attention reads it */
  size_t o_offset;          /* [T, Lq]: attention output, heads concatenated */
  size_t wo_offset;         /* [E, Lq]: W_o in the intermediate type */
  size_t wc_offset;         /* [n_q + n_kv, d, d]: channel-conv weights (q heads, then K heads) in the
                               intermediate type */
  size_t sched_offset;      /* scratch of the attention kernel: split-pair counters and partial rows */
} cca_workspace_layout_t;

/* Checks a configuration. CCA_OK if some kernel path accepts it. */
cca_status_t cca_validate(const cca_config_t* cfg);

/* Workspace bytes that cca_prefill needs for cfg (0 if cfg is invalid). */
size_t cca_workspace_size(const cca_config_t* cfg);

/* Kernel choice of cca_prefill_ex(cfg, ..., path) on the current device. */
cca_status_t cca_plan(const cca_config_t* cfg, int path, cca_plan_t* out);

/* Fills *out with the workspace layout for cfg. */
cca_status_t cca_workspace_layout(const cca_config_t* cfg, cca_workspace_layout_t* out);

/*
 * Prefill forward of one CCA / CCGQA block over B sequences of S tokens.
 *
 * Inputs (device, cfg->dtype, Lq = n_q*d, Lkv = n_kv*d, T = B*S):
 *   x          [B, S, E]         hidden states
 *   W_q        [Lq, E]           down-projections (torch Linear layout)
 *   W_k, W_v   [Lkv, E]
 *   convq_seq  [Lq, K]           causal seq-conv taps per q channel; tap K-1
 *                                multiplies the current token
 *   convq_chan [n_q, d, d]       per-head channel mix: out_i = sum_j W[i][j] in_j
 *   convk_seq  [Lkv, K], convk_chan [n_kv, d, d]   the same for k
 *   W_o        [E, Lq]           output projection
 * Outputs (device):
 *   y          [B, S, E]         cfg->out_dtype
 *   k_cache    [B, S, n_kv, d]   k after convs, QK-mean and RoPE
 *   v_cache    [B, S, n_kv, d]   v after the value shift
 *   conv_state optional (NULL to skip), [B, (K-1)*(Lq+Lkv) + Lkv]: per
 *              sequence the last K-1 rows of q~ (each Lq wide), then of k~
 *              (Lkv wide), then the last row of v~; rows before the sequence
 *              start are zero. It is what a later decode step would resume
 *              from.
 *   workspace  >= cca_workspace_size(cfg) bytes, 256-byte aligned; holds the
 *              intermediates listed in cca_workspace_layout_t.
 * Errors: INVALID_ARG / UNSUPPORTED / WORKSPACE before any launch; CUDA if a
 * launch fails. A device-side wait that gives up is reported later by
 * cca_poll_device_status.
 */
cca_status_t cca_prefill(const cca_config_t* cfg,
                         const void* x,
                         const void* W_q, const void* W_k, const void* W_v,
                         const void* convq_seq, const void* convq_chan,
                         const void* convk_seq, const void* convk_chan,
                         const void* W_o,
                         void* y, void* k_cache, void* v_cache, void* conv_state,
                         void* workspace, size_t workspace_bytes, void* stream);

/* cca_prefill with options (path choice, per-stage events); opts may be NULL. */
cca_status_t cca_prefill_ex(const cca_config_t* cfg,
                            const void* x,
                            const void* W_q, const void* W_k, const void* W_v,
                            const void* convq_seq, const void* convq_chan,
                            const void* convk_seq, const void* convk_chan,
                            const void* W_o,
                            void* y, void* k_cache, void* v_cache, void* conv_state,
                            void* workspace, size_t workspace_bytes, void* stream,
                            const cca_prefill_opts_t* opts);

/*
 * End-to-end variant for callers whose hidden states live in host memory:
 * copies x_host (B*S*E elements, pinned host memory for a truly asynchronous
 * copy) into the device buffer x_dev, runs cca_prefill, and copies y back
 * from y_dev into y_host (pinned). The KV cache stays on the device. All
 * three steps are enqueued on `stream`; y_host is valid once the stream has
 * been synchronized.
 */
cca_status_t cca_prefill_host(const cca_config_t* cfg,
                              const void* x_host, void* x_dev,
                              const void* W_q, const void* W_k, const void* W_v,
                              const void* convq_seq, const void* convq_chan,
                              const void* convk_seq, const void* convk_chan,
                              const void* W_o,
                              void* y_dev, void* y_host,
                              void* k_cache, void* v_cache, void* conv_state,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * cca_prefill without a caller-provided workspace. The paper has no
 * counterpart; this exists for callers that must not allocate device memory
 * while they run: cudaMalloc can synchronize the device and stall every
 * stream of the process, runtimes that own the whole device memory pool (and
 * the plugins they host) forbid it, and a caller that already holds all of its
 * memory has nowhere to get cca_workspace_size() bytes from.
 *
 * The intermediates go to a fixed 256-byte-aligned device array inside the
 * library of CCA_NOALLOC_WORKSPACE_BYTES; every GPU on which this is called
 * keeps that memory until the process exits (under lazy module loading, the
 * default of recent CUDA runtimes; with CUDA_MODULE_LOADING=EAGER every GPU on
 * which the library is loaded reserves it, whether or not this is called). Blocks whose
 * cca_workspace_size() exceeds it are rejected with CCA_ERR_WORKSPACE (e.g.
 * B=1, S=8192, E=2048, 4 query / 2 KV heads of 128 needs 44 MB and fits;
 * S=16384 does not). The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress); make that first call before capturing a
 * stream. All calls share the array: calls whose work may overlap on the GPU
 * (other streams, other host threads on the device) race on it, so order them.
 * Nothing in it needs to start at zero. Arguments, outputs and errors are
 * those of cca_prefill; the library allocates nothing.
 */
#define CCA_NOALLOC_WORKSPACE_BYTES 67108864
cca_status_t cca_prefill_noalloc(const cca_config_t* cfg,
                                 const void* x,
                                 const void* W_q, const void* W_k, const void* W_v,
                                 const void* convq_seq, const void* convq_chan,
                                 const void* convk_seq, const void* convk_chan,
                                 const void* W_o,
                                 void* y, void* k_cache, void* v_cache, void* conv_state,
                                 void* stream);

/*
 * One decode step of the block ("Compressed Convolutional Attention",
 * gist.science/es/paper/2510.04476, section 1 item 2: decoding reads the
 * compressed KV cache, C times smaller than a multi-head one; the steps are
 * those of the prefill, section 2, for one more token): the token at position
 * t = cfg->seq_len - 1 of each of the cfg->batch sequences, given the state a
 * cca_prefill of tokens 0..t-1 (or earlier decode steps) left. All sequences
 * are at the same position. Arithmetic is fp32; inputs, weights, the cache
 * and the conv state are cfg->dtype.
 *
 *   cache_rows  rows allocated per sequence in k_cache / v_cache, >= seq_len
 *   x_t         [B, E]                 hidden state of the new token
 *   W_q ... W_o as in cca_prefill (the conv weights may be NULL when K == 0)
 *   y_t         [B, E] out             cfg->out_dtype
 *   k_cache, v_cache [B, cache_rows, n_kv, d] in/out: rows 0..t-1 are read,
 *               row t is written. A prefill writes [B, S, n_kv, d]; with
 *               B > 1 its rows must be copied into the wider cache first.
 *   conv_state  [B, (K-1)*(Lq+Lkv) + Lkv] in/out, as cca_prefill writes it;
 *               advanced by one token in place. Required when K >= 1, NULL
 *               when K == 0.
 *   workspace   >= cca_decode_workspace_size(cfg) bytes, 256-byte aligned,
 *               need not start at zero. The size does not depend on seq_len,
 *               so one buffer serves every step.
 * Supported: head_dim 32, 64 or 128; n_q_heads / n_kv_heads <= 8; hidden and
 * n_q_heads * head_dim multiples of 8; all pointers 16-byte aligned.
 * Launches 4 kernels (3 when K == 0) for B <= 8, and two more per further 8
 * sequences. Errors: INVALID_ARG / UNSUPPORTED / WORKSPACE before any launch,
 * CUDA if a launch fails. No kernel of this step waits on another.
 */
size_t cca_decode_workspace_size(const cca_config_t* cfg);
cca_status_t cca_decode(const cca_config_t* cfg, int cache_rows,
                        const void* x_t,
                        const void* W_q, const void* W_k, const void* W_v,
                        const void* convq_seq, const void* convq_chan,
                        const void* convk_seq, const void* convk_chan,
                        const void* W_o,
                        void* y_t, void* k_cache, void* v_cache, void* conv_state,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * The backward pass of one block ("Compressed Convolutional Attention",
 * gist.science/es/paper/2510.04476: section 4 times the backward of CCGQA;
 * what it computes is the chain rule through the forward of section 2 taken
 * in reverse): given dy = dL/dy, the gradient of L with respect to x and to
 * every weight, for the same inputs as cca_prefill.
 *
 * The forward's activations are recomputed first, by the forward's own
 * kernels (the path AUTO picks), into the workspace. Then, for bf16 blocks
 * with head_dim 128 on sm_100, the attention backward, the channel-mix
 * backward and the projection gradients run on the tensor cores: fp16 or
 * bf16 operands, and fp32 values that bf16 does not hold exactly split into
 * bf16 high and low parts, all accumulating in fp32. The remaining
 * transposes (RoPE, QK-mean, value shift, sequence conv) run in fp32 on the
 * CUDA cores. Other blocks run every step in fp32 on the CUDA cores. The
 * reductions over tokens use atomic fp32 additions, so repeated calls agree
 * to rounding, not bit for bit.
 *
 *   x ... W_o   as in cca_prefill, cfg->dtype
 *   dy          [B, S, E]              cfg->out_dtype
 *   dx          [B, S, E] out          fp32
 *   dW_q        [Lq, E] out, dW_k and dW_v [Lkv, E] out     fp32
 *   dconvq_seq  [Lq, K], dconvq_chan [n_q, d, d] out        fp32
 *   dconvk_seq  [Lkv, K], dconvk_chan [n_kv, d, d] out      fp32
 *   dW_o        [E, Lq] out            fp32
 *   workspace   >= cca_backward_workspace_size(cfg) bytes, 256-byte aligned,
 *               need not start at zero
 * Every output is overwritten (not accumulated). Supported: conv_kernel 0..8
 * (a plain block, conv_kernel 0, takes NULL for the four conv weights and
 * their gradients), even head_dim <= 128, (n_q_heads + n_kv_heads) * head_dim
 * <= 12288, dtype bf16 or fp32, and what cca_prefill supports for cfg; all
 * pointers 16-byte aligned, no output aliasing another buffer.
 * cca_backward_workspace_size returns 0 for an unsupported or invalid cfg.
 * Errors: INVALID_ARG / UNSUPPORTED / WORKSPACE before any launch, CUDA if a
 * launch fails; device-side conditions (an fp16 intermediate of the forward
 * out of range, a bounded wait that gave up) through cca_poll_device_status.
 */
size_t cca_backward_workspace_size(const cca_config_t* cfg);
cca_status_t cca_backward(const cca_config_t* cfg,
                          const void* x,
                          const void* W_q, const void* W_k, const void* W_v,
                          const void* convq_seq, const void* convq_chan,
                          const void* convk_seq, const void* convk_chan,
                          const void* W_o, const void* dy,
                          float* dx, float* dW_q, float* dW_k, float* dW_v,
                          float* dconvq_seq, float* dconvq_chan,
                          float* dconvk_seq, float* dconvk_chan, float* dW_o,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * A training step's forward and backward without recomputing the forward:
 * cca_prefill_train runs the block like cca_prefill (same inputs; y, k_cache
 * and v_cache written) and keeps in `workspace` (>= cca_backward_workspace_size
 * bytes, 256-byte aligned) the intermediates and each attention row's
 * log-sum-exp that the backward reads. cca_backward_saved then computes the
 * gradients of cca_backward from that workspace, skipping the forward: the
 * caller passes the same cfg, inputs and workspace, and nothing may have
 * written the workspace in between (the results are those of cca_backward).
 * For bf16 blocks whose attention runs on the tensor cores (sm_100, head_dim
 * 128); other blocks return CCA_ERR_UNSUPPORTED from both (use cca_prefill
 * and cca_backward). Errors and pointer rules as cca_prefill / cca_backward;
 * cca_prefill_train takes no conv state.
 */
cca_status_t cca_prefill_train(const cca_config_t* cfg,
                               const void* x,
                               const void* W_q, const void* W_k, const void* W_v,
                               const void* convq_seq, const void* convq_chan,
                               const void* convk_seq, const void* convk_chan,
                               const void* W_o,
                               void* y, void* k_cache, void* v_cache,
                               void* workspace, size_t workspace_bytes, void* stream);
cca_status_t cca_backward_saved(const cca_config_t* cfg,
                                const void* x,
                                const void* W_q, const void* W_k, const void* W_v,
                                const void* convq_seq, const void* convq_chan,
                                const void* convk_seq, const void* convk_chan,
                                const void* W_o, const void* dy,
                                float* dx, float* dW_q, float* dW_k, float* dW_v,
                                float* dconvq_seq, float* dconvq_chan,
                                float* dconvk_seq, float* dconvk_chan, float* dW_o,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Synchronizes `stream`, then reports and clears the device error word:
 * CCA_ERR_DEVICE_TIMEOUT if a bounded wait in a kernel gave up since the last
 * poll, CCA_ERR_NUMERIC_RANGE if a finite fp16 intermediate overflowed (its
 * stored value is then +-inf), CCA_ERR_CUDA if the stream reports a CUDA
 * error, else CCA_OK. */
cca_status_t cca_poll_device_status(void* stream);

/* Self-test of the bounded-wait machinery: launches one kernel that waits on
 * an mbarrier nothing will ever complete, with a limit of `timeout_us`
 * microseconds (1..5000000). The kernel gives up, records the timeout in the
 * device error word and exits; cca_poll_device_status then returns
 * CCA_ERR_DEVICE_TIMEOUT. */
cca_status_t cca_selftest_wait_timeout(unsigned timeout_us, void* stream);

/* Static description of a status code. */
const char* cca_status_string(cca_status_t status);

/* One-line reason for the last non-OK status returned on this host thread. */
const char* cca_last_error_message(void);

/* CCA_VERSION of the built library. */
int cca_version(void);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* CCA_H_ */
