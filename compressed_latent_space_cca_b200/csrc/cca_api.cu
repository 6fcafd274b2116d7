// C ABI of the CCA / CCGQA prefill library: validation, workspace layout,
// path choice and the launch sequence
//   down-projection -> preprocessing -> attention -> output projection
// of one block ("Compressed Convolutional Attention", gist.science/es/paper/
// 2510.04476, section 2). Every step runs in this library's kernels.
#include <math.h>
#include <stdio.h>

#include <mutex>
#include <string>

#include "../../include/cca.h"
#include "cca_common.cuh"
#include "launch.h"

namespace cca {

// Device error word, set by bounded waits that give up.
__device__ unsigned g_device_error = 0;

namespace {

thread_local std::string t_last_error;

cca_status_t fail(cca_status_t st, const std::string& msg) {
  t_last_error = msg;
  return st;
}

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct DeviceInfo {
  bool init = false;
  int major = 0, minor = 0, sms = 0;
  unsigned* err_ptr = nullptr;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

cca_status_t device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(CCA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(CCA_ERR_UNSUPPORTED, "device index out of range");
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.init) {
    cudaDeviceProp prop;
    if ((e = cudaGetDeviceProperties(&prop, dev)) != cudaSuccess)
      return fail(CCA_ERR_CUDA, std::string("cudaGetDeviceProperties: ") + cudaGetErrorString(e));
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_device_error)) != cudaSuccess)
      return fail(CCA_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    di.major = prop.major;
    di.minor = prop.minor;
    di.sms = prop.multiProcessorCount;
    di.err_ptr = static_cast<unsigned*>(p);
    di.init = true;
  }
  *out = &di;
  return CCA_OK;
}

bool is_dtype(int v) { return v == CCA_F32 || v == CCA_BF16; }

cca_status_t check_config(const cca_config_t* c, BlockDims* dm) {
  if (c == nullptr) return fail(CCA_ERR_INVALID_ARG, "cfg is NULL");
  if (c->batch < 1 || c->seq_len < 1 || c->hidden < 1)
    return fail(CCA_ERR_INVALID_ARG, "batch, seq_len and hidden must be >= 1");
  if (c->n_q_heads < 1 || c->n_kv_heads < 1) return fail(CCA_ERR_INVALID_ARG, "head counts must be >= 1");
  if (c->n_q_heads % c->n_kv_heads != 0)
    return fail(CCA_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads");
  if (c->head_dim < 2 || c->head_dim % 2 != 0) return fail(CCA_ERR_INVALID_ARG, "head_dim must be even and >= 2");
  if (c->C < 1) return fail(CCA_ERR_INVALID_ARG, "C must be >= 1");
  if ((long long)c->C * c->n_q_heads * c->head_dim != c->hidden)
    return fail(CCA_ERR_INVALID_ARG, "hidden must equal C * n_q_heads * head_dim");
  if (c->conv_kernel < 0 || c->conv_kernel > 64) return fail(CCA_ERR_INVALID_ARG, "conv_kernel must be in [0, 64]");
  if (c->conv_kernel == 0 && (c->qk_mean_mode != 0 || c->value_shift != 0))
    return fail(CCA_ERR_INVALID_ARG, "a plain block (conv_kernel 0) takes qk_mean_mode 0 and value_shift 0");
  if (c->qk_mean_mode < 0 || c->qk_mean_mode > 3) return fail(CCA_ERR_INVALID_ARG, "qk_mean_mode must be in [0, 3]");
  if (c->value_shift != 0 && c->value_shift != 1) return fail(CCA_ERR_INVALID_ARG, "value_shift must be 0 or 1");
  if (c->use_rope != 0 && c->use_rope != 1) return fail(CCA_ERR_INVALID_ARG, "use_rope must be 0 or 1");
  if (c->use_rope && !(c->rope_base > 1.0f && isfinite(c->rope_base)))
    return fail(CCA_ERR_INVALID_ARG, "rope_base must be finite and > 1");
  if (!(c->softmax_scale >= 0.0f) || !isfinite(c->softmax_scale))
    return fail(CCA_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  if (!is_dtype(c->dtype) || !is_dtype(c->out_dtype)) return fail(CCA_ERR_INVALID_ARG, "unknown dtype");
  {
    const long long lkv = (long long)c->n_kv_heads * c->head_dim;
    if (c->kv_channel_offset < 0 || c->kv_total_channels < 0 || c->kv_channel_offset % 8 != 0 ||
        c->kv_total_channels % 16 != 0 ||
        (c->kv_total_channels > 0 && c->kv_total_channels < c->kv_channel_offset + lkv) ||
        (c->kv_total_channels == 0 && c->kv_channel_offset != 0))
      return fail(CCA_ERR_INVALID_ARG,
                  "kv_channel_offset must be a multiple of 8 and kv_total_channels a multiple of 16 that holds "
                  "this block's V channels past the offset (both 0 for a whole block)");
  }
  if (c->head_dim > 128) return fail(CCA_ERR_UNSUPPORTED, "head_dim > 128 is not supported");
  const long long T = (long long)c->batch * c->seq_len;
  const long long Nlat = (long long)(c->n_q_heads + 2 * c->n_kv_heads) * c->head_dim;
  if (T > (1ll << 30) || Nlat > (1 << 20) || c->hidden > (1 << 20))
    return fail(CCA_ERR_UNSUPPORTED, "tensor extent too large");
  if (dm) {
    dm->B = c->batch;
    dm->S = c->seq_len;
    dm->E = c->hidden;
    dm->nq = c->n_q_heads;
    dm->nkv = c->n_kv_heads;
    dm->d = c->head_dim;
    dm->K = c->conv_kernel;
    dm->G = c->n_q_heads / c->n_kv_heads;
    dm->Lq = c->n_q_heads * c->head_dim;
    dm->Lkv = c->n_kv_heads * c->head_dim;
    dm->Nlat = dm->Lq + 2 * dm->Lkv;
    dm->T = T;
    dm->qk_mean_mode = c->qk_mean_mode;
    dm->value_shift = c->value_shift;
    {
      const long long total = c->kv_total_channels > 0 ? c->kv_total_channels : (long long)dm->Lkv;
      long long from = total / 2 - c->kv_channel_offset;
      from = from < 0 ? 0 : (from > dm->Lkv ? dm->Lkv : from);
      dm->vshift_from = (int)from;
    }
    dm->use_rope = c->use_rope;
    dm->rope_base = c->rope_base;
    dm->scale = c->softmax_scale > 0.f ? c->softmax_scale : 1.0f / sqrtf((float)c->head_dim);
    dm->io = c->dtype == CCA_BF16 ? DType::BF16 : DType::F32;
    dm->lat = c->dtype == CCA_BF16 ? DType::F16 : DType::F32;
    dm->out = c->out_dtype == CCA_BF16 ? DType::BF16 : DType::F32;
  }
  return CCA_OK;
}

cca_workspace_layout_t layout_of(const BlockDims& dm) {
  cca_workspace_layout_t L;
  const size_t eb = dtype_bytes(dm.lat);
  const bool sep = dm.lat != dm.io;  // attention K/V and W_o need their own copies
  L.elem_bytes = eb;
  L.lat_dtype = dm.lat == DType::F16 ? CCA_F16 : (dm.lat == DType::BF16 ? CCA_BF16 : CCA_F32);
  size_t off = 0;
  L.qkv_lat_offset = off;
  off = align_up(off + (size_t)dm.T * dm.Nlat * eb);
  L.q_offset = off;
  off = align_up(off + (size_t)dm.T * dm.Lq * eb);
  L.k_att_offset = off;
  if (sep) off = align_up(off + (size_t)dm.T * dm.Lkv * eb);
  L.v_att_offset = off;
  if (sep) off = align_up(off + (size_t)dm.T * dm.Lkv * eb);
  L.o_offset = off;
  off = align_up(off + (size_t)dm.T * dm.Lq * eb);
  L.wo_offset = off;
  if (sep) off = align_up(off + (size_t)dm.E * dm.Lq * eb);
  L.wc_offset = off;
  if (sep && dm.K > 0) off = align_up(off + (size_t)(dm.nq + dm.nkv) * dm.d * dm.d * eb);
  L.sched_offset = off;
  off = align_up(off + (attention_tc_supported(dm) ? attention_tc_scratch_bytes(dm) : 256));
  L.total_bytes = off;
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Resolved {
  BlockDims dm;
  bool tc_down, tc_attn, tc_out;  // tcgen05 kernels per stage
  bool tc_pre;                    // tensor-core preprocessing kernel (mma.sync form)
  bool pre_ws;                    // tensor-core preprocessing kernel (warp-specialised tcgen05 form)
  bool v_fuse;                    // value shift in the down-projection's epilogue (with pre_ws)
};

cca_status_t resolve(const cca_config_t* cfg, int path, Resolved* r) {
  cca_status_t st = check_config(cfg, &r->dm);
  if (st != CCA_OK) return st;
  DeviceInfo* di = nullptr;
  if ((st = device_info(&di)) != CCA_OK) return st;
  const BlockDims& dm = r->dm;
  const bool masked = (path & ~63) == CCA_PATH_TENSOR_MASK(0);
  if (path != CCA_PATH_AUTO && path != CCA_PATH_SIMT && path != CCA_PATH_TENSOR && !masked)
    return fail(CCA_ERR_INVALID_ARG, "unknown path");
  const bool sm100 = di->major == 10;
  const bool b16 = dm.io == DType::BF16;
  const bool down = sm100 && b16 && gemm_tc_supported(dm.T, dm.Nlat, dm.E) && dm.Lq % 128 == 0 &&
                    dm.Lkv % 128 == 0;
  const bool attn = sm100 && b16 && dm.d == 128 && attention_tc_supported(dm);
  const bool out = sm100 && b16 && gemm_tc_supported(dm.T, dm.E, dm.Lq);
  const bool pre = preproc_tc_supported(dm);
  const bool ws = sm100 && preproc_ws_supported(dm);
  if (path == CCA_PATH_TENSOR && !(down && attn && out && (pre || dm.K == 0)))
    return fail(CCA_ERR_UNSUPPORTED, "tensor-core path needs sm_100, bf16, head_dim 128 and 128-aligned widths");
  if (masked && (((path & 1) && !down) || ((path & 2) && !attn) || ((path & 4) && !out) || ((path & 8) && !pre) ||
                 ((path & 16) && !ws)))
    return fail(CCA_ERR_UNSUPPORTED, "a stage asked for the tensor-core kernel cannot use it");
  if (masked && (path & 8) && (path & 16))
    return fail(CCA_ERR_INVALID_ARG, "path bits 3 and 4 both choose the preprocessing kernel");
  if (masked && (path & 32) && !((path & 1) && (path & 16)))
    return fail(CCA_ERR_INVALID_ARG, "path bit 5 (value shift in the down-projection) needs bits 0 and 4");
  const bool use = path != CCA_PATH_SIMT;
  r->tc_down = masked ? (path & 1) != 0 : use && down;
  r->tc_attn = masked ? (path & 2) != 0 : use && attn;
  r->tc_out = masked ? (path & 4) != 0 : use && out;
  // AUTO takes the warp-specialised tcgen05 preprocessing where it applies (the QK-mean includes the
  // after-conv term), else the mma.sync kernel; TENSOR keeps the mma.sync kernel
  r->pre_ws = masked ? (path & 16) != 0 : (path == CCA_PATH_AUTO && ws);
  r->tc_pre = masked ? (path & 8) != 0 : use && pre && !r->pre_ws;
  r->v_fuse = masked && (path & 32) != 0;
  return CCA_OK;
}

cca_status_t cuda_fail(const char* what, cudaError_t e) {
  return fail(CCA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

cca_status_t run_block(const Resolved& r, BlockPtrs p, cudaStream_t stream, void* const* ev) {
  const BlockDims& dm = r.dm;
  DeviceInfo* di = nullptr;
  cca_status_t st = device_info(&di);
  if (st != CCA_OK) return st;
  p.dev_err = di->err_ptr;
  cudaError_t e;
  auto mark = [&](int i) -> cudaError_t {
    return ev ? cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), stream) : cudaSuccess;
  };
  const size_t eb = dtype_bytes(dm.lat);
  if ((e = mark(0)) != cudaSuccess) return cuda_fail("event", e);
  // 1. down-projection: q~ | k~ | v~ = x [W_q; W_k; W_v]^T
  if (r.tc_down) {
    GemmTcArgs a{};
    a.A = p.x;
    a.M = dm.T;
    a.K = dm.E;
    a.B[0] = p.Wq;
    a.B[1] = p.Wk;
    a.B[2] = p.Wv;
    a.nrows[0] = dm.Lq;
    a.nrows[1] = dm.Lkv;
    a.nrows[2] = dm.Lkv;
    a.nb = 3;
    a.C = p.qkv_lat;
    a.ldc = dm.Nlat;
    a.in = dm.io;
    a.out = dm.lat;
    a.dev_err = p.dev_err;
    if (r.tc_pre || r.pre_ws) {  // the fp16 channel-conv weights of the preprocessing kernel, made on the side
      const long long nc = (long long)dm.d * dm.d;
      a.side_scale = r.pre_ws ? kWsWeightScale : 1.0f;
      if (p.v_fused) {  // v~ leaves the epilogue as the value-shifted V cache and its attention copy
        a.v_cache = p.v_cache;
        a.v_att = p.v_att;
        a.v_col0 = dm.Lq + dm.Lkv;
        a.Lkv = dm.Lkv;
        a.S = dm.S;
        a.vshift = dm.value_shift;
        a.vfrom = dm.vshift_from;
      }
      a.side_src[0] = p.cq_chan;
      a.side_dst[0] = p.wc_lat;
      a.side_n[0] = nc * dm.nq;
      a.side_src[1] = p.ck_chan;
      a.side_dst[1] = static_cast<char*>(p.wc_lat) + nc * dm.nq * eb;
      a.side_n[1] = nc * dm.nkv;
    }
    if ((e = launch_gemm_tc(a, stream)) != cudaSuccess) return cuda_fail("down-projection (tcgen05)", e);
  } else {
    char* out = static_cast<char*>(p.qkv_lat);
    const void* Ws[3] = {p.Wq, p.Wk, p.Wv};
    const int ns[3] = {dm.Lq, dm.Lkv, dm.Lkv};
    int col = 0;
    for (int i = 0; i < 3; ++i) {
      if ((e = launch_gemm_simt(dm.io, dm.lat, p.x, dm.E, Ws[i], dm.E, out + (size_t)col * eb, dm.Nlat, dm.T,
                                ns[i], dm.E, stream, p.dev_err)) != cudaSuccess)
        return cuda_fail("down-projection (SIMT)", e);
      col += ns[i];
    }
    if (r.tc_pre || r.pre_ws) {
      const long long nc = (long long)dm.d * dm.d;
      const float sc = r.pre_ws ? kWsWeightScale : 1.0f;
      if ((e = launch_convert_f16(p.cq_chan, p.wc_lat, nc * dm.nq, p.dev_err, stream, sc)) != cudaSuccess ||
          (e = launch_convert_f16(p.ck_chan, static_cast<char*>(p.wc_lat) + nc * dm.nq * eb, nc * dm.nkv, p.dev_err,
                                  stream, sc)) != cudaSuccess)
        return cuda_fail("channel-conv weight copy", e);
    }
  }
  if ((e = mark(1)) != cudaSuccess) return cuda_fail("event", e);
  // 2. seq conv, channel conv, QK-mean, RoPE, value shift; KV cache written here
  if (dm.K == 0) {
    if ((e = launch_plain_preproc(dm, p, stream)) != cudaSuccess) return cuda_fail("RoPE and KV cache (plain)", e);
  } else if (r.pre_ws) {
    if ((e = launch_preproc_ws(dm, p, stream)) != cudaSuccess) return cuda_fail("preprocessing (tcgen05)", e);
  } else if (r.tc_pre) {
    if ((e = launch_preproc_tc(dm, p, stream)) != cudaSuccess) return cuda_fail("preprocessing (mma)", e);
  } else {
    if ((e = launch_preproc_simt(dm, p, stream)) != cudaSuccess) return cuda_fail("preprocessing (SIMT)", e);
  }
  if ((e = launch_conv_state(dm, p, stream)) != cudaSuccess) return cuda_fail("conv state", e);
  if ((e = mark(2)) != cudaSuccess) return cuda_fail("event", e);
  // 3. causal attention on the compressed heads
  if (r.tc_attn) {
    if ((e = launch_attention_tc(dm, p.q, p.k_att, p.v_att, p.o, p.sched, p.dev_err, stream, p.lse2,
                                 p.lse_stride)) != cudaSuccess)
      return cuda_fail("attention (tcgen05)", e);
  } else {
    if ((e = launch_attention_simt(dm, p.q, p.k_att, p.v_att, p.o, stream)) != cudaSuccess)
      return cuda_fail("attention (SIMT)", e);
  }
  if ((e = mark(3)) != cudaSuccess) return cuda_fail("event", e);
  // 4. output projection y = o W_o^T
  if (r.tc_out) {
    GemmTcArgs a{};
    a.A = p.o;
    a.M = dm.T;
    a.K = dm.Lq;
    a.B[0] = p.wo_lat;
    a.nrows[0] = dm.E;
    a.nb = 1;
    a.C = p.y;
    a.ldc = dm.E;
    a.in = dm.lat;
    a.out = dm.out;
    a.dev_err = p.dev_err;
    if ((e = launch_gemm_tc(a, stream)) != cudaSuccess) return cuda_fail("output projection (tcgen05)", e);
  } else {
    if ((e = launch_gemm_simt(dm.lat, dm.out, p.o, dm.Lq, p.wo_lat, dm.Lq, p.y, dm.E, dm.T, dm.E, dm.Lq, stream,
                              p.dev_err)) != cudaSuccess)
      return cuda_fail("output projection (SIMT)", e);
  }
  if ((e = mark(4)) != cudaSuccess) return cuda_fail("event", e);
  return CCA_OK;
}

cca_status_t prepare(const cca_config_t* cfg, int path, const void* const* ins, void* const* outs, void* conv_state,
                     void* workspace, size_t workspace_bytes, Resolved* r, BlockPtrs* p) {
  cca_status_t st = resolve(cfg, path, r);
  if (st != CCA_OK) return st;
  static const char* in_names[9] = {"x", "W_q", "W_k", "W_v", "convq_seq", "convq_chan", "convk_seq", "convk_chan",
                                    "W_o"};
  const bool plain = r->dm.K == 0;  // no convolutions: their weights may be NULL
  for (int i = 0; i < 9; ++i) {
    if (plain && i >= 4 && i <= 7 && ins[i] == nullptr) continue;
    if (ins[i] == nullptr) return fail(CCA_ERR_INVALID_ARG, std::string(in_names[i]) + " is NULL");
    if (!aligned16(ins[i])) return fail(CCA_ERR_INVALID_ARG, std::string(in_names[i]) + " is not 16-byte aligned");
  }
  static const char* out_names[3] = {"y", "k_cache", "v_cache"};
  for (int i = 0; i < 3; ++i) {
    if (outs[i] == nullptr) return fail(CCA_ERR_INVALID_ARG, std::string(out_names[i]) + " is NULL");
    if (!aligned16(outs[i])) return fail(CCA_ERR_INVALID_ARG, std::string(out_names[i]) + " is not 16-byte aligned");
  }
  if (conv_state != nullptr && !aligned16(conv_state))
    return fail(CCA_ERR_INVALID_ARG, "conv_state is not 16-byte aligned");
  if (conv_state != nullptr && plain) return fail(CCA_ERR_INVALID_ARG, "a plain block (conv_kernel 0) has no conv state");
  const cca_workspace_layout_t L = layout_of(r->dm);
  if (workspace == nullptr) return fail(CCA_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(CCA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (workspace_bytes < L.total_bytes)
    return fail(CCA_ERR_WORKSPACE, "workspace smaller than cca_workspace_size()");
  char* ws = static_cast<char*>(workspace);
  p->x = ins[0];
  p->Wq = ins[1];
  p->Wk = ins[2];
  p->Wv = ins[3];
  p->cq_seq = ins[4];
  p->cq_chan = ins[5];
  p->ck_seq = ins[6];
  p->ck_chan = ins[7];
  p->Wo = ins[8];
  p->y = outs[0];
  p->k_cache = outs[1];
  p->v_cache = outs[2];
  p->conv_state = conv_state;
  const bool sep = r->dm.lat != r->dm.io;
  p->qkv_lat = ws + L.qkv_lat_offset;
  p->q = ws + L.q_offset;
  p->k_att = sep ? ws + L.k_att_offset : outs[1];
  p->v_att = sep ? ws + L.v_att_offset : outs[2];
  p->o = ws + L.o_offset;
  p->wo_lat = sep ? ws + L.wo_offset : const_cast<void*>(ins[8]);
  p->wc_lat = sep ? ws + L.wc_offset : nullptr;
  p->sched = ws + L.sched_offset;
  p->dev_err = nullptr;
  p->lse2 = nullptr;
  p->lse_stride = 0;
  // the conv state keeps the last v~ row, which the fused value shift does not write; the fused
  // epilogue shifts whole 64-channel groups
  p->v_fused = r->v_fuse && conv_state == nullptr && r->dm.vshift_from % 64 == 0;
  return CCA_OK;
}

}  // namespace

int set_last_error(int status, const char* msg) {
  t_last_error = msg;
  return status;
}

int num_sms() {
  DeviceInfo* di = nullptr;
  if (device_info(&di) != CCA_OK) return 148;
  return di->sms;
}

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// -------------------------------------------------------- self-test kernel --
namespace {
__global__ void wait_timeout_selftest_kernel(unsigned* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t a = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(a, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on this barrier: the bounded wait must give up.
  if (threadIdx.x == 0) (void)mbar_wait_bounded(a, 0, err, nullptr, wait_site(kSiteSelftest, 0, 0), limit_ns);
}
}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned* dev_err, unsigned long long limit_ns, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(dev_err, limit_ns);
  return cudaGetLastError();
}

}  // namespace cca

// ============================================================== C ABI ==
using namespace cca;

extern "C" {

int cca_version(void) { return CCA_VERSION; }

const char* cca_status_string(cca_status_t s) {
  switch (s) {
    case CCA_OK: return "ok";
    case CCA_ERR_INVALID_ARG: return "invalid argument";
    case CCA_ERR_UNSUPPORTED: return "unsupported configuration";
    case CCA_ERR_WORKSPACE: return "workspace missing or too small";
    case CCA_ERR_CUDA: return "CUDA error";
    case CCA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case CCA_ERR_NUMERIC_RANGE: return "intermediate out of fp16 range";
  }
  return "unknown status";
}

const char* cca_last_error_message(void) { return t_last_error.c_str(); }

cca_status_t cca_validate(const cca_config_t* cfg) {
  BlockDims dm;
  cca_status_t st = check_config(cfg, &dm);
  if (st == CCA_OK) t_last_error.clear();
  return st;
}

size_t cca_workspace_size(const cca_config_t* cfg) {
  BlockDims dm;
  if (check_config(cfg, &dm) != CCA_OK) return 0;
  return layout_of(dm).total_bytes;
}

cca_status_t cca_plan(const cca_config_t* cfg, int path, cca_plan_t* out) {
  if (out == nullptr) return fail(CCA_ERR_INVALID_ARG, "out is NULL");
  Resolved r;
  cca_status_t st = resolve(cfg, path, &r);
  if (st != CCA_OK) return st;
  out->down_proj_tensor = r.tc_down;
  out->attention_tensor = r.tc_attn;
  out->out_proj_tensor = r.tc_out;
  out->preproc_tensor = r.pre_ws ? 2 : (r.tc_pre ? 1 : 0);
  out->value_shift_fused = r.v_fuse;
  // down-projection (one tcgen05 GEMM, or three SIMT GEMMs plus the two fp16 weight copies that the
  // tcgen05 GEMM otherwise makes on the side), preprocessing, attention, output projection
  out->launches = (r.tc_down ? 1 : 3 + (r.tc_pre || r.pre_ws ? 2 : 0)) + 1 + 1 + 1;
  return CCA_OK;
}

cca_status_t cca_workspace_layout(const cca_config_t* cfg, cca_workspace_layout_t* out) {
  if (out == nullptr) return fail(CCA_ERR_INVALID_ARG, "out is NULL");
  BlockDims dm;
  cca_status_t st = check_config(cfg, &dm);
  if (st != CCA_OK) return st;
  *out = layout_of(dm);
  return CCA_OK;
}

cca_status_t cca_prefill_ex(const cca_config_t* cfg, const void* x, const void* W_q, const void* W_k,
                            const void* W_v, const void* convq_seq, const void* convq_chan, const void* convk_seq,
                            const void* convk_chan, const void* W_o, void* y, void* k_cache, void* v_cache,
                            void* conv_state, void* workspace, size_t workspace_bytes, void* stream,
                            const cca_prefill_opts_t* opts) {
  const void* ins[9] = {x, W_q, W_k, W_v, convq_seq, convq_chan, convk_seq, convk_chan, W_o};
  void* outs[3] = {y, k_cache, v_cache};
  Resolved r;
  BlockPtrs p;
  const int path = opts ? opts->path : CCA_PATH_AUTO;
  cca_status_t st = prepare(cfg, path, ins, outs, conv_state, workspace, workspace_bytes, &r, &p);
  if (st != CCA_OK) return st;
  return run_block(r, p, static_cast<cudaStream_t>(stream), opts ? opts->stage_events : nullptr);
}

cca_status_t cca_prefill(const cca_config_t* cfg, const void* x, const void* W_q, const void* W_k, const void* W_v,
                         const void* convq_seq, const void* convq_chan, const void* convk_seq,
                         const void* convk_chan, const void* W_o, void* y, void* k_cache, void* v_cache,
                         void* conv_state, void* workspace, size_t workspace_bytes, void* stream) {
  return cca_prefill_ex(cfg, x, W_q, W_k, W_v, convq_seq, convq_chan, convk_seq, convk_chan, W_o, y, k_cache,
                        v_cache, conv_state, workspace, workspace_bytes, stream, nullptr);
}

cca_status_t cca_prefill_host(const cca_config_t* cfg, const void* x_host, void* x_dev, const void* W_q,
                              const void* W_k, const void* W_v, const void* convq_seq, const void* convq_chan,
                              const void* convk_seq, const void* convk_chan, const void* W_o, void* y_dev,
                              void* y_host, void* k_cache, void* v_cache, void* conv_state, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (x_host == nullptr || y_host == nullptr) return fail(CCA_ERR_INVALID_ARG, "host buffer is NULL");
  const void* ins[9] = {x_dev, W_q, W_k, W_v, convq_seq, convq_chan, convk_seq, convk_chan, W_o};
  void* outs[3] = {y_dev, k_cache, v_cache};
  Resolved r;
  BlockPtrs p;
  cca_status_t st = prepare(cfg, CCA_PATH_AUTO, ins, outs, conv_state, workspace, workspace_bytes, &r, &p);
  if (st != CCA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t xbytes = (size_t)r.dm.T * r.dm.E * dtype_bytes(r.dm.io);
  const size_t ybytes = (size_t)r.dm.T * r.dm.E * dtype_bytes(r.dm.out);
  cudaError_t e = cudaMemcpyAsync(x_dev, x_host, xbytes, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail("copy x to device", e);
  if ((st = run_block(r, p, s, nullptr)) != CCA_OK) return st;
  e = cudaMemcpyAsync(y_host, y_dev, ybytes, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail("copy y to host", e);
  return CCA_OK;
}

size_t cca_decode_workspace_size(const cca_config_t* cfg) {
  BlockDims dm;
  if (check_config(cfg, &dm) != CCA_OK || !decode_supported(dm)) return 0;
  return decode_workspace_bytes(dm);
}

cca_status_t cca_decode(const cca_config_t* cfg, int cache_rows, const void* x_t, const void* W_q, const void* W_k,
                        const void* W_v, const void* convq_seq, const void* convq_chan, const void* convk_seq,
                        const void* convk_chan, const void* W_o, void* y_t, void* k_cache, void* v_cache,
                        void* conv_state, void* workspace, size_t workspace_bytes, void* stream) {
  BlockDims dm;
  cca_status_t st = check_config(cfg, &dm);
  if (st != CCA_OK) return st;
  if (!decode_supported(dm))
    return fail(CCA_ERR_UNSUPPORTED,
                "decode needs head_dim 32, 64 or 128, n_q_heads / n_kv_heads <= 8, hidden and n_q_heads * "
                "head_dim multiples of 8");
  if (cache_rows < dm.S) return fail(CCA_ERR_INVALID_ARG, "cache_rows must be >= seq_len");
  if ((long long)dm.B * cache_rows > (1ll << 30)) return fail(CCA_ERR_UNSUPPORTED, "cache extent too large");
  static const char* names[10] = {"x_t", "W_q", "W_k", "W_v", "convq_seq", "convq_chan", "convk_seq", "convk_chan",
                                  "W_o", "y_t"};
  const void* ptrs[10] = {x_t, W_q, W_k, W_v, convq_seq, convq_chan, convk_seq, convk_chan, W_o, y_t};
  const bool plain = dm.K == 0;
  for (int i = 0; i < 10; ++i) {
    if (plain && i >= 4 && i <= 7 && ptrs[i] == nullptr) continue;
    if (ptrs[i] == nullptr) return fail(CCA_ERR_INVALID_ARG, std::string(names[i]) + " is NULL");
    if (!aligned16(ptrs[i])) return fail(CCA_ERR_INVALID_ARG, std::string(names[i]) + " is not 16-byte aligned");
  }
  if (k_cache == nullptr || v_cache == nullptr) return fail(CCA_ERR_INVALID_ARG, "k_cache / v_cache is NULL");
  if (!aligned16(k_cache) || !aligned16(v_cache))
    return fail(CCA_ERR_INVALID_ARG, "k_cache / v_cache is not 16-byte aligned");
  if (plain && conv_state != nullptr)
    return fail(CCA_ERR_INVALID_ARG, "a plain block (conv_kernel 0) has no conv state");
  if (!plain && conv_state == nullptr) return fail(CCA_ERR_INVALID_ARG, "conv_state is NULL");
  if (workspace == nullptr) return fail(CCA_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(CCA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (workspace_bytes < decode_workspace_bytes(dm))
    return fail(CCA_ERR_WORKSPACE, "workspace smaller than cca_decode_workspace_size()");
  DecodePtrs p{x_t, W_q, W_k, W_v, convq_seq, convq_chan, convk_seq, convk_chan, W_o,
               y_t, k_cache, v_cache, conv_state, workspace};
  const cudaError_t e = launch_decode(dm, p, cache_rows, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail("decode", e);
  return CCA_OK;
}

size_t cca_backward_workspace_size(const cca_config_t* cfg) {
  BlockDims dm;
  if (check_config(cfg, &dm) != CCA_OK || !backward_supported(dm)) return 0;
  return backward_layout(dm, layout_of(dm).total_bytes).total;
}

}  // extern "C"

namespace {
// The three ways a backward call or its forward run: the backward with the forward recomputed into
// its workspace (RECOMPUTE), a forward that keeps what a later backward reads (KEEP: y, the KV
// cache and, in the workspace, the intermediates and the rows' log-sum-exp), and the backward from
// such a workspace (SAVED).
enum class BwdMode { RECOMPUTE, KEEP, SAVED };

cca_status_t backward_call(BwdMode mode, const cca_config_t* cfg, const void* const* ins, const void* dy, float* const* gp9,
                           void* const* outs3, void* workspace, size_t workspace_bytes, void* stream) {
  BlockDims dm;
  cca_status_t st = check_config(cfg, &dm);
  if (st != CCA_OK) return st;
  if (!backward_supported(dm))
    return fail(CCA_ERR_UNSUPPORTED,
                "backward needs conv_kernel 0..8, an even head_dim <= 128, n_q_heads + n_kv_heads times head_dim "
                "<= 12288 and bf16 or fp32");
  const bool plain = dm.K == 0;  // no convolutions: their weights and gradients may be NULL
  if (mode != BwdMode::KEEP) {
    static const char* g_names[10] = {"dy",         "dx",          "dW_q",       "dW_k",        "dW_v",
                                      "dconvq_seq", "dconvq_chan", "dconvk_seq", "dconvk_chan", "dW_o"};
    const void* gp[10] = {dy, gp9[0], gp9[1], gp9[2], gp9[3], gp9[4], gp9[5], gp9[6], gp9[7], gp9[8]};
    for (int i = 0; i < 10; ++i) {
      if (plain && i >= 5 && i <= 8 && gp[i] == nullptr) continue;
      if (gp[i] == nullptr) return fail(CCA_ERR_INVALID_ARG, std::string(g_names[i]) + " is NULL");
      if (!aligned16(gp[i])) return fail(CCA_ERR_INVALID_ARG, std::string(g_names[i]) + " is not 16-byte aligned");
    }
  }
  static const char* in_names[9] = {"x", "W_q", "W_k", "W_v", "convq_seq", "convq_chan", "convk_seq", "convk_chan",
                                    "W_o"};
  for (int i = 0; i < 9; ++i) {
    if (plain && i >= 4 && i <= 7 && ins[i] == nullptr) continue;
    if (ins[i] == nullptr) return fail(CCA_ERR_INVALID_ARG, std::string(in_names[i]) + " is NULL");
    if (!aligned16(ins[i])) return fail(CCA_ERR_INVALID_ARG, std::string(in_names[i]) + " is not 16-byte aligned");
  }
  if (workspace == nullptr) return fail(CCA_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(CCA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  const size_t fwd = layout_of(dm).total_bytes;
  const BackwardLayout BL = backward_layout(dm, fwd);
  if (workspace_bytes < BL.total) return fail(CCA_ERR_WORKSPACE, "workspace smaller than cca_backward_workspace_size()");
  char* ws = static_cast<char*>(workspace);
  void* inner[3] = {ws + BL.y, ws + BL.k_cache, ws + BL.v_cache};
  Resolved r;
  BlockPtrs p;
  if ((st = prepare(cfg, CCA_PATH_AUTO, ins, mode == BwdMode::KEEP ? outs3 : inner, nullptr, workspace, fwd, &r, &p)) !=
      CCA_OK)
    return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the tensor-core attention backward reads the log-sum-exp rows the forward's attention leaves
  const bool tc_bwd = r.tc_attn && attention_bwd_tc_supported(r.dm);
  // a saved forward lives in the workspace only where its attention operands are the workspace's own
  // copies and the log-sum-exp rows exist: bf16 blocks on the tensor-core attention
  if (mode != BwdMode::RECOMPUTE && !(tc_bwd && r.dm.lat != r.dm.io))
    return fail(CCA_ERR_UNSUPPORTED,
                "a saved forward needs a bf16 block on the tensor-core attention (use cca_backward otherwise)");
  if (tc_bwd) {
    p.lse2 = reinterpret_cast<float*>(ws + BL.lse);
    p.lse_stride = BL.stat_stride;
  }
  if (mode != BwdMode::SAVED && (st = run_block(r, p, s, nullptr)) != CCA_OK) return st;
  if (mode == BwdMode::KEEP) return CCA_OK;
  DeviceInfo* di = nullptr;
  if ((st = device_info(&di)) != CCA_OK) return st;
  p.dev_err = di->err_ptr;  // the backward kernels' bounded waits and range checks report here
  const BackwardPtrs g{dy, gp9[0], gp9[1], gp9[2], gp9[3], gp9[4], gp9[5], gp9[6], gp9[7], gp9[8]};
  const cudaError_t e = launch_backward(r.dm, p, g, BL, ws, s, tc_bwd, r.tc_down && r.tc_out);
  if (e != cudaSuccess) return cuda_fail("backward", e);
  return CCA_OK;
}
}  // namespace

extern "C" {

cca_status_t cca_backward(const cca_config_t* cfg, const void* x, const void* W_q, const void* W_k, const void* W_v,
                          const void* convq_seq, const void* convq_chan, const void* convk_seq,
                          const void* convk_chan, const void* W_o, const void* dy, float* dx, float* dW_q,
                          float* dW_k, float* dW_v, float* dconvq_seq, float* dconvq_chan, float* dconvk_seq,
                          float* dconvk_chan, float* dW_o, void* workspace, size_t workspace_bytes, void* stream) {
  const void* ins[9] = {x, W_q, W_k, W_v, convq_seq, convq_chan, convk_seq, convk_chan, W_o};
  float* g[9] = {dx, dW_q, dW_k, dW_v, dconvq_seq, dconvq_chan, dconvk_seq, dconvk_chan, dW_o};
  return backward_call(BwdMode::RECOMPUTE, cfg, ins, dy, g, nullptr, workspace, workspace_bytes, stream);
}

cca_status_t cca_prefill_train(const cca_config_t* cfg, const void* x, const void* W_q, const void* W_k,
                               const void* W_v, const void* convq_seq, const void* convq_chan, const void* convk_seq,
                               const void* convk_chan, const void* W_o, void* y, void* k_cache, void* v_cache,
                               void* workspace, size_t workspace_bytes, void* stream) {
  const void* ins[9] = {x, W_q, W_k, W_v, convq_seq, convq_chan, convk_seq, convk_chan, W_o};
  void* outs[3] = {y, k_cache, v_cache};
  return backward_call(BwdMode::KEEP, cfg, ins, nullptr, nullptr, outs, workspace, workspace_bytes, stream);
}

cca_status_t cca_backward_saved(const cca_config_t* cfg, const void* x, const void* W_q, const void* W_k,
                                const void* W_v, const void* convq_seq, const void* convq_chan, const void* convk_seq,
                                const void* convk_chan, const void* W_o, const void* dy, float* dx, float* dW_q,
                                float* dW_k, float* dW_v, float* dconvq_seq, float* dconvq_chan, float* dconvk_seq,
                                float* dconvk_chan, float* dW_o, void* workspace, size_t workspace_bytes,
                                void* stream) {
  const void* ins[9] = {x, W_q, W_k, W_v, convq_seq, convq_chan, convk_seq, convk_chan, W_o};
  float* g[9] = {dx, dW_q, dW_k, dW_v, dconvq_seq, dconvq_chan, dconvk_seq, dconvk_chan, dW_o};
  return backward_call(BwdMode::SAVED, cfg, ins, dy, g, nullptr, workspace, workspace_bytes, stream);
}

cca_status_t cca_poll_device_status(void* stream) {
  DeviceInfo* di = nullptr;
  cca_status_t st = device_info(&di);
  if (st != CCA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail("stream synchronize", e);
  unsigned h = 0;
  if ((e = cudaMemcpy(&h, di->err_ptr, sizeof(h), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail("read device error word", e);
  if (h != 0) {
    unsigned zero = 0;
    if ((e = cudaMemcpy(di->err_ptr, &zero, sizeof(zero), cudaMemcpyHostToDevice)) != cudaSuccess)
      return cuda_fail("clear device error word", e);
    if ((h & 0xffu) == kDevErrRange)
      return fail(CCA_ERR_NUMERIC_RANGE, "an intermediate exceeded the fp16 range (|value| > 65504)");
    static const char* kernels[8] = {"?",         "gemm", "attention", "self-test", "?", "preprocessing (tcgen05)",
                                     "attention backward", "channel-mix backward"};
    char msg[160];
    snprintf(msg, sizeof(msg), "a bounded device-side wait gave up (kernel %s, role %u, barrier %u)",
             kernels[((h >> 8) & 0xffu) < 8 ? ((h >> 8) & 0xffu) : 0], (h >> 16) & 0xffu, (h >> 24) & 0xffu);
    return fail(CCA_ERR_DEVICE_TIMEOUT, msg);
  }
  return CCA_OK;
}

cca_status_t cca_selftest_wait_timeout(unsigned timeout_us, void* stream) {
  if (timeout_us < 1 || timeout_us > 5000000u) return fail(CCA_ERR_INVALID_ARG, "timeout_us must be in [1, 5e6]");
  DeviceInfo* di = nullptr;
  cca_status_t st = device_info(&di);
  if (st != CCA_OK) return st;
  cudaError_t e = launch_wait_timeout_selftest(di->err_ptr, (unsigned long long)timeout_us * 1000ull,
                                               static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail("self-test launch", e);
  return CCA_OK;
}

}  // extern "C"
