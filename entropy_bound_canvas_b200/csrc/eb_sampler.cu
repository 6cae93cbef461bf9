// eb_sampler.cu -- host side of the C ABI declared in include/eb_sampler.h.
//
// Validation, the device workspace, launch configuration and error codes.
// A step is one kernel on the caller's stream: the persistent stream kernel
// (eb_stream.cuh, one CTA per SM: every logit once, every position's
// entropy, argmax, max probability and draw, and each canvas's decisions),
// launched as a programmatic dependent of the stream's previous kernel so
// that its set-up overlaps that kernel's end.  All the per-step arithmetic
// runs in the kernels.
#include "eb_sampler.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <mutex>
#include <new>

#include <cudaTypedefs.h>

#include "eb_finish.cuh"
#include "eb_lmhead.cuh"
#include "eb_stream.cuh"

namespace {

using ebk::Rec;
using ebk::StepArgs;

struct KernelCfg {
  const void* fn = nullptr;
  size_t smem = 0;
  int grid = 0;
};

constexpr int kMaxDevices = 64;

// Kernel attributes are process-wide per device: the stream kernels'
// dynamic shared memory opt-in is set once per device to the device maximum,
// so that no handle ever lowers a value another handle relies on.
struct DeviceAttrs {
  std::once_flag once;
  int rc = EB_ERR_CUDA;
  int sms = 0;
  size_t optin = 0;
};
DeviceAttrs g_dev[kMaxDevices];

void device_setup(DeviceAttrs& d, int device) {
  int sms = 0, optin = 0, major = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess) {
    cudaGetLastError();
    d.rc = EB_ERR_CUDA;
    return;
  }
  if (major != 10) {
    d.rc = EB_ERR_UNSUPPORTED;
    return;
  }
  if (cudaFuncSetAttribute(ebk::stream_kernel<ebk::kF32>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, optin) != cudaSuccess ||
      cudaFuncSetAttribute(ebk::stream_kernel<ebk::kBF16>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, optin) != cudaSuccess ||
      cudaFuncSetAttribute(ebk::combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin) != cudaSuccess ||
      cudaFuncSetAttribute(ebk::lmhead_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin) != cudaSuccess ||
      cudaFuncSetAttribute(ebk::lmhead_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin) != cudaSuccess) {
    cudaGetLastError();
    d.rc = EB_ERR_CUDA;
    return;
  }
  d.sms = sms;
  d.optin = (size_t)optin;
  d.rc = EB_OK;
}

// The current device's attributes, set up on first use (the device must be
// current).
int device_attrs(int device, DeviceAttrs** out) {
  if (device < 0 || device >= kMaxDevices) return EB_ERR_UNSUPPORTED;
  DeviceAttrs& d = g_dev[device];
  std::call_once(d.once, device_setup, std::ref(d), device);
  *out = &d;
  return d.rc;
}

}  // namespace

struct eb_sampler {
  eb_config_t cfg;
  int device = 0;
  int sms = 0;
  int ng = 0;
  int max_segs = 0;  // stream CTAs that can share one row
  KernelCfg k[2];    // stream kernel [dtype]
  KernelCfg combine;  // combine kernel (vocabulary slices)
  int V_tot = 0;      // global vocabulary size
  int slice_step = -1;
  uint64_t wait_ns = ebk::kWaitLimitNs;
  // workspace (one allocation)
  void* ws = nullptr;
  size_t ws_bytes = 0;
  Rec* recs = nullptr;
  int32_t* row_cnt = nullptr;
  int32_t* canvas_cnt = nullptr;
  int32_t* sync_cnt = nullptr;
  uint32_t* status = nullptr;
  int32_t* act_index = nullptr;
  int32_t* n_act = nullptr;
  int32_t* prev_amax = nullptr;
  int32_t* stable = nullptr;
  int32_t* sample = nullptr;
  float* pmax = nullptr;
  int last_step = -1;
  cudaEvent_t split_event = nullptr;  // recorded after the step's kernel when set
  // the LM-head step's per-(position, vocabulary range) records
  ebk::SliceRecord* lm_rec = nullptr;
  int lm_split = 0;
};

namespace {

// Restores the caller's current device on scope exit.
struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && cudaSetDevice(dev) == cudaSuccess) ok = true;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

int validate_config(const eb_config_t* c) {
  if (!c) return EB_ERR_INVALID_ARG;
  if (c->B < 1 || c->L < 1 || c->V < 1 || c->num_steps < 1) return EB_ERR_INVALID_ARG;
  if (c->B > EB_MAX_CANVASES || c->L > EB_MAX_POSITIONS) return EB_ERR_OVERFLOW;
  if (c->canvas_offset < 0 || (int64_t)c->canvas_offset + c->B > (int64_t)(1 << 24))
    return EB_ERR_OVERFLOW;
  if (c->rule != EB_RULE_ENTROPY_BOUND && c->rule != EB_RULE_BLOCK_REFINEMENT &&
      c->rule != EB_RULE_ENTROPY_BOUND_MI)
    return EB_ERR_INVALID_ARG;
  if (c->greedy != 0 && c->greedy != 1) return EB_ERR_INVALID_ARG;
  if (!c->greedy && !(c->t_max > 0.0 && c->t_min > 0.0 && std::isfinite(c->t_max) &&
                      std::isfinite(c->t_min)))
    return EB_ERR_INVALID_ARG;
  if (!(c->entropy_bound >= 0.0) || !std::isfinite(c->entropy_bound)) return EB_ERR_INVALID_ARG;
  if (std::isnan(c->stop_entropy) || std::isnan(c->threshold) || std::isnan(c->editing_threshold))
    return EB_ERR_INVALID_ARG;
  if (c->stability_steps < 0 || c->quota < 0) return EB_ERR_INVALID_ARG;
  // a vocabulary slice starts on a group boundary and lies inside the vocabulary
  if (c->vocab_offset < 0 || c->vocab_offset % ebk::kGroup != 0 || c->vocab_total < 0)
    return EB_ERR_INVALID_ARG;
  if (c->vocab_total > 0 && (int64_t)c->vocab_offset + c->V > (int64_t)c->vocab_total)
    return EB_ERR_INVALID_ARG;
  if (c->vocab_total == 0 && c->vocab_offset != 0) return EB_ERR_INVALID_ARG;
  // group numbering fits the 64-bit work split: B * L * ng * grid < 2^63
  const uint64_t ng = ((uint64_t)c->V + ebk::kGroup - 1) / ebk::kGroup;
  if ((uint64_t)c->B * (uint64_t)c->L * ng >= (1ull << 46)) return EB_ERR_OVERFLOW;
  return EB_OK;
}

// One persistent CTA per SM, fewer if there are fewer stage-sized tiles.
template <int DT>
int stream_grid(int sms, uint64_t groups) {
  const uint64_t want = (groups + ebk::StreamShape<DT>::kStageGroups - 1) /
                        ebk::StreamShape<DT>::kStageGroups;
  return (int)std::min<uint64_t>((uint64_t)sms, std::max<uint64_t>(1, want));
}

// Most stream CTAs one row can span when each owns at least
// floor(rows ng / G) groups: floor((ng - 1) G / (rows ng)) + 2, at most G.
int row_max_segs(int G, uint64_t rows, int ng) {
  const uint64_t Lng = rows * (uint64_t)ng;
  const uint64_t segs = ((uint64_t)(ng - 1) * (uint64_t)G) / Lng + 2;
  return (int)std::min<uint64_t>((uint64_t)G, segs);
}

template <int DT>
int setup_kernel(eb_sampler* h, const DeviceAttrs& d) {
  KernelCfg& kc = h->k[DT];
  kc.fn = reinterpret_cast<const void*>(&ebk::stream_kernel<DT>);
  kc.smem = ebk::stream_layout<DT>(h->cfg.B).total;
  if (kc.smem > d.optin) return EB_ERR_OVERFLOW;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ebk::stream_kernel<DT>,
                                                    ebk::StreamShape<DT>::kThreads, kc.smem) !=
          cudaSuccess ||
      per_sm < 1)
    return EB_ERR_CUDA;
  const uint64_t groups = (uint64_t)h->cfg.B * (uint64_t)h->cfg.L * (uint64_t)h->ng;
  kc.grid = stream_grid<DT>(d.sms, groups);
  return EB_OK;
}

}  // namespace

extern "C" {

void eb_config_default(eb_config_t* cfg, int32_t B, int32_t L, int32_t V) {
  if (!cfg) return;
  std::memset(cfg, 0, sizeof(*cfg));
  cfg->B = B;
  cfg->L = L;
  cfg->V = V;
  cfg->num_steps = 48;
  cfg->t_max = 0.8;
  cfg->t_min = 0.4;
  cfg->entropy_bound = 0.1;
  cfg->stop_entropy = 0.005;
  cfg->stability_steps = 1;
  cfg->rule = EB_RULE_ENTROPY_BOUND;
  cfg->threshold = 0.9;
  cfg->quota = (L + 47) / 48;
  cfg->greedy = 0;
  cfg->canvas_offset = 0;
  cfg->seed = 0;
  cfg->editing_threshold = -1.0;
  cfg->vocab_offset = 0;
  cfg->vocab_total = 0;
}

int eb_sampler_init(eb_sampler_t** out, const eb_config_t* cfg, int device) {
  if (!out) return EB_ERR_INVALID_ARG;
  *out = nullptr;
  int rc = validate_config(cfg);
  if (rc != EB_OK) return rc;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess) return EB_ERR_CUDA;
  if (device < 0 || device >= ndev) return EB_ERR_INVALID_ARG;
  DeviceGuard guard(device);
  if (!guard.ok) return EB_ERR_CUDA;
  DeviceAttrs* d = nullptr;
  if ((rc = device_attrs(device, &d)) != EB_OK) return rc;

  eb_sampler* h = new (std::nothrow) eb_sampler();
  if (!h) return EB_ERR_OUT_OF_MEMORY;
  h->cfg = *cfg;
  h->device = device;
  h->sms = d->sms;
  h->ng = (int)(((int64_t)cfg->V + ebk::kGroup - 1) / ebk::kGroup);

  if ((rc = setup_kernel<ebk::kF32>(h, *d)) != EB_OK ||
      (rc = setup_kernel<ebk::kBF16>(h, *d)) != EB_OK) {
    delete h;
    return rc;
  }
  h->combine.fn = reinterpret_cast<const void*>(&ebk::combine_kernel);
  h->combine.smem = ebk::epi_layout(cfg->L).total;
  h->combine.grid = cfg->B;
  if (h->combine.smem > d->optin) {
    delete h;
    return EB_ERR_OVERFLOW;
  }
  h->V_tot = cfg->vocab_total > 0 ? cfg->vocab_total : cfg->V;
  int gmax = 0;
  for (int k = 0; k < 2; ++k) gmax = std::max(gmax, h->k[k].grid);
  h->max_segs = row_max_segs(gmax, (uint64_t)cfg->L, h->ng);

  const size_t BL = (size_t)cfg->B * (size_t)cfg->L;
  size_t off = 0;
  const size_t o_rec = off;
  off = align256(off + sizeof(Rec) * BL * (size_t)h->max_segs);
  const size_t o_cnt = off;
  off = align256(off + sizeof(int32_t) * BL);
  const size_t o_ccnt = off;
  off = align256(off + sizeof(int32_t) * (size_t)cfg->B);
  const size_t o_sync = off;
  off = align256(off + sizeof(int32_t) * 2);
  const size_t o_status = off;
  off = align256(off + sizeof(uint32_t));
  const size_t o_act = off;
  off = align256(off + sizeof(int32_t) * ((size_t)cfg->B + 1));
  const size_t o_prev = off;
  off = align256(off + sizeof(int32_t) * BL);
  const size_t o_stable = off;
  off = align256(off + sizeof(int32_t) * (size_t)cfg->B);
  const size_t o_sample = off;
  off = align256(off + sizeof(int32_t) * BL);
  const size_t o_pmax = off;
  off = align256(off + sizeof(float) * BL);
  h->ws_bytes = off;
  if (cudaMalloc(&h->ws, h->ws_bytes) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return EB_ERR_OUT_OF_MEMORY;
  }
  if (cudaMemset(h->ws, 0, h->ws_bytes) != cudaSuccess) {
    cudaFree(h->ws);
    delete h;
    return EB_ERR_CUDA;
  }
  char* base = static_cast<char*>(h->ws);
  h->recs = reinterpret_cast<Rec*>(base + o_rec);
  h->row_cnt = reinterpret_cast<int32_t*>(base + o_cnt);
  h->canvas_cnt = reinterpret_cast<int32_t*>(base + o_ccnt);
  h->sync_cnt = reinterpret_cast<int32_t*>(base + o_sync);
  h->status = reinterpret_cast<uint32_t*>(base + o_status);
  h->act_index = reinterpret_cast<int32_t*>(base + o_act);
  h->n_act = h->act_index + cfg->B;
  h->prev_amax = reinterpret_cast<int32_t*>(base + o_prev);
  h->stable = reinterpret_cast<int32_t*>(base + o_stable);
  h->sample = reinterpret_cast<int32_t*>(base + o_sample);
  h->pmax = reinterpret_cast<float*>(base + o_pmax);
  *out = h;
  return EB_OK;
}

int eb_sampler_init_canvas(eb_sampler_t* h, int32_t* canvas, uint8_t* committed,
                           uint8_t* stop_flags, void* stream) {
  if (!h || !canvas || !committed || !stop_flags) return EB_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok) return EB_ERR_CUDA;
  const eb_config_t& c = h->cfg;
  ebk::init_canvas_kernel<<<c.B, 256, 0, (cudaStream_t)stream>>>(
      canvas, committed, stop_flags, h->stable, h->row_cnt, h->canvas_cnt, c.L, h->V_tot,
      c.canvas_offset,
      (uint32_t)(c.seed & 0xffffffffu), (uint32_t)(c.seed >> 32));
  if (cudaGetLastError() != cudaSuccess) return EB_ERR_CUDA;
  h->last_step = -1;
  h->slice_step = -1;
  return EB_OK;
}

}  // extern "C"

namespace {

// Temperature of step s: linear from t_max to t_min over num_steps (T = 1
// when greedy).
double step_temperature(const eb_config_t& c, int step) {
  return c.greedy ? 1.0
         : c.num_steps <= 1
             ? c.t_max
             : c.t_max + (c.t_min - c.t_max) * (double)step / (double)(c.num_steps - 1);
}

// The step's arguments that do not depend on the caller's buffers.
void fill_args(const eb_sampler* h, StepArgs& a, int step) {
  const eb_config_t& c = h->cfg;
  const double T = step_temperature(c, step);
  std::memset(&a, 0, sizeof(a));
  a.recs = h->recs;
  a.row_cnt = h->row_cnt;
  a.canvas_cnt = h->canvas_cnt;
  a.sync_cnt = h->sync_cnt;
  a.prev_amax = h->prev_amax;
  a.stable = h->stable;
  a.sample = h->sample;
  a.pmax = h->pmax;
  a.status = h->status;
  a.act_index = h->act_index;
  a.n_act = h->n_act;
  a.wait_ns = h->wait_ns;
  a.B = c.B;
  a.L = c.L;
  a.V = c.V;
  a.ng = h->ng;
  a.s = step;
  a.N = c.num_steps;
  a.max_segs = h->max_segs;
  a.rule = c.rule;
  a.quota = c.quota;
  a.stability_steps = c.stability_steps;
  a.greedy = c.greedy;
  a.stop_enabled = c.stop_entropy >= 0.0 ? 1 : 0;
  a.canvas_offset = c.canvas_offset;
  a.c2 = (float)(1.4426950408889634 / T);
  a.iT = (float)(1.0 / T);
  a.gamma = c.entropy_bound;
  a.tau = c.stop_entropy;
  a.theta = c.threshold;
  a.eps_edit = c.rule == EB_RULE_BLOCK_REFINEMENT ? c.editing_threshold : -1.0;
  a.v_off = c.vocab_offset;
  a.V_tot = h->V_tot;
  a.key0 = (uint32_t)(c.seed & 0xffffffffu);
  a.key1 = (uint32_t)(c.seed >> 32);
}

// A kernel launched as a programmatic dependent of the previous one on `st`.
int launch_dependent(const void* fn, dim3 grid, dim3 block, size_t smem, void** args,
                     cudaStream_t st) {
  cudaLaunchConfig_t lc;
  std::memset(&lc, 0, sizeof(lc));
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelExC(&lc, fn, args) == cudaSuccess ? EB_OK : EB_ERR_CUDA;
}

// The stream kernel over `logits` (this device's rows or vocabulary slice),
// a programmatic dependent of the stream's previous kernel.
int launch_stream(const KernelCfg& kc, StepArgs& a, const void* logits, int dtype, size_t V,
                  cudaStream_t st) {
  const size_t elt = dtype == EB_F32 ? 4 : 2;
  a.logits = logits;
  a.vec_ok = ((uintptr_t)logits % 16 == 0) && ((V * elt) % 16 == 0) ? 1 : 0;
  a.G1 = kc.grid;
  void* args[] = {&a};
  return launch_dependent(kc.fn, dim3(kc.grid), dim3(ebk::stream_threads(dtype)), kc.smem, args,
                          st);
}

bool is_slice(const eb_sampler* h) {
  return h->cfg.vocab_offset != 0 || h->V_tot != h->cfg.V;
}

// ---------------------------------------------------------------------------
// LM-head step: tensor maps and launch
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    cudaGetLastError();
  });
  return fn;
}

// A bf16 matrix [outer][inner] (inner contiguous), read in boxes of
// box_outer x 64 with the 128-byte swizzle the MMA descriptors expect.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
               uint32_t box_outer) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tmap_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {(cuuint32_t)ebk::kLmBK, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Sizes the LM-head kernels accept: the hidden size a multiple of 64, the
// vocabulary a multiple of 256 (one MMA N tile), 16-byte aligned operands.
int lm_check(const void* hidden, const void* weight, int64_t rows, int64_t V, int64_t d) {
  if (!hidden || !weight || rows < 1 || V < ebk::kLmBN || d < ebk::kLmBK)
    return EB_ERR_INVALID_ARG;
  if (d % ebk::kLmBK != 0 || V % ebk::kLmBN != 0) return EB_ERR_UNSUPPORTED;
  if ((uintptr_t)hidden % 16 != 0 || (uintptr_t)weight % 16 != 0) return EB_ERR_INVALID_ARG;
  if (rows > (1ll << 30) || V > (1ll << 30) || d > (1 << 20)) return EB_ERR_OVERFLOW;
  return EB_OK;
}

// Vocabulary ranges per 128-row tile: one CTA per SM over all tiles.
int lm_split_count(int sms, int64_t rows, int64_t V) {
  const int n_mt = (int)((rows + ebk::kLmBM - 1) / ebk::kLmBM);
  const int n_nt = (int)(V / ebk::kLmBN);
  return std::max(1, std::min(n_nt, sms / std::max(1, n_mt)));
}

int lm_launch(bool sampler, const DeviceAttrs& d, const void* hidden, const void* weight,
              ebk::LmArgs& p, cudaStream_t st) {
  CUtensorMap th, tw;
  if (!make_tmap(&th, hidden, (uint64_t)p.d, (uint64_t)p.rows, ebk::kLmBM) ||
      !make_tmap(&tw, weight, (uint64_t)p.d, (uint64_t)p.V, ebk::kLmBN))
    return EB_ERR_CUDA;
  const size_t smem = ebk::lm_layout(sampler).total;
  if (smem > d.optin) return EB_ERR_UNSUPPORTED;
  const int n_mt = (p.rows + ebk::kLmBM - 1) / ebk::kLmBM;
  void* args[] = {&th, &tw, &p};
  const void* fn = sampler ? reinterpret_cast<const void*>(&ebk::lmhead_kernel<true>)
                           : reinterpret_cast<const void*>(&ebk::lmhead_kernel<false>);
  if (cudaLaunchKernel(fn, dim3(n_mt * p.n_split), dim3(ebk::kLmThreads), args, smem, st) !=
      cudaSuccess)
    return EB_ERR_CUDA;
  return EB_OK;
}

}  // namespace

extern "C" {

int eb_sampler_step(eb_sampler_t* h, const void* logits, int dtype, int step, int32_t* canvas,
                    uint8_t* committed, float* entropies, int32_t* argmax, uint8_t* stop_flags,
                    void* stream) {
  if (!h || !logits || !canvas || !committed || !entropies || !argmax || !stop_flags)
    return EB_ERR_INVALID_ARG;
  if (dtype != EB_F32 && dtype != EB_BF16) return EB_ERR_UNSUPPORTED;
  if ((uintptr_t)logits % (dtype == EB_F32 ? 4u : 2u) != 0) return EB_ERR_INVALID_ARG;
  if (is_slice(h)) return EB_ERR_INVALID_ARG;  // a vocabulary slice steps by slice + combine
  const eb_config_t& c = h->cfg;
  if (step < 0 || step >= c.num_steps) return EB_ERR_INVALID_ARG;
  if (step != 0 && step != h->last_step + 1) return EB_ERR_STEP_ORDER;
  DeviceGuard guard(h->device);
  if (!guard.ok) return EB_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;

  StepArgs a;
  fill_args(h, a, step);
  a.canvas = canvas;
  a.committed = committed;
  a.H_out = entropies;
  a.amax_out = argmax;
  a.stop_flags = stop_flags;
  a.run_epilogue = 1;
  const int rc = launch_stream(h->k[dtype], a, logits, dtype, (size_t)c.V, st);
  if (rc != EB_OK) return rc;
  if (h->split_event && cudaEventRecord(h->split_event, st) != cudaSuccess) return EB_ERR_CUDA;
  h->last_step = step;
  return EB_OK;
}

int eb_sampler_step_slice(eb_sampler_t* h, const void* logits, int dtype, int step,
                          const uint8_t* committed, const uint8_t* stop_flags, void* records,
                          void* stream) {
  if (!h || !logits || !committed || !stop_flags || !records) return EB_ERR_INVALID_ARG;
  if (dtype != EB_F32 && dtype != EB_BF16) return EB_ERR_UNSUPPORTED;
  if ((uintptr_t)logits % (dtype == EB_F32 ? 4u : 2u) != 0 || (uintptr_t)records % 8 != 0)
    return EB_ERR_INVALID_ARG;
  const eb_config_t& c = h->cfg;
  if (step < 0 || step >= c.num_steps) return EB_ERR_INVALID_ARG;
  if (step != 0 && step != h->slice_step + 1) return EB_ERR_STEP_ORDER;
  DeviceGuard guard(h->device);
  if (!guard.ok) return EB_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;

  StepArgs a;
  fill_args(h, a, step);
  a.committed = const_cast<uint8_t*>(committed);  // read only on this path
  a.stop_flags = const_cast<uint8_t*>(stop_flags);
  a.slice_out = static_cast<ebk::SliceRecord*>(records);
  const int rc = launch_stream(h->k[dtype], a, logits, dtype, (size_t)c.V, st);
  if (rc != EB_OK) return rc;
  h->slice_step = step;
  return EB_OK;
}

int eb_sampler_combine(eb_sampler_t* h, const void* records, int n_slices, int step,
                       int32_t* canvas, uint8_t* committed, float* entropies, int32_t* argmax,
                       uint8_t* stop_flags, void* stream) {
  if (!h || !records || !canvas || !committed || !entropies || !argmax || !stop_flags ||
      n_slices < 1 || (uintptr_t)records % 8 != 0)
    return EB_ERR_INVALID_ARG;
  const eb_config_t& c = h->cfg;
  if (step < 0 || step >= c.num_steps) return EB_ERR_INVALID_ARG;
  if (step != 0 && step != h->last_step + 1) return EB_ERR_STEP_ORDER;
  if (h->slice_step != step) return EB_ERR_STEP_ORDER;  // this handle's slice of the step first
  DeviceGuard guard(h->device);
  if (!guard.ok) return EB_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;

  StepArgs a;
  fill_args(h, a, step);
  a.canvas = canvas;
  a.committed = committed;
  a.H_out = entropies;
  a.amax_out = argmax;
  a.stop_flags = stop_flags;
  const int32_t* act_index = h->act_index;
  const ebk::SliceRecord* rec = static_cast<const ebk::SliceRecord*>(records);
  void* cargs[] = {&a, &act_index, &rec, &n_slices};
  if (cudaLaunchKernel(h->combine.fn, dim3(h->combine.grid), dim3(ebk::kEpiThreads), cargs,
                       h->combine.smem, st) != cudaSuccess)
    return EB_ERR_CUDA;
  h->last_step = step;
  return EB_OK;
}

size_t eb_slice_record_bytes(void) { return sizeof(ebk::SliceRecord); }

int eb_lmhead_logits(const void* hidden, const void* weight, int32_t rows, int32_t V, int32_t d,
                     float* logits, void* stream) {
  int rc = lm_check(hidden, weight, rows, V, d);
  if (rc != EB_OK) return rc;
  if (!logits || (uintptr_t)logits % 16 != 0) return EB_ERR_INVALID_ARG;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return EB_ERR_CUDA;
  DeviceAttrs* da = nullptr;
  if ((rc = device_attrs(device, &da)) != EB_OK) return rc;
  ebk::LmArgs p;
  std::memset(&p, 0, sizeof(p));
  p.a.wait_ns = ebk::kWaitLimitNs;
  p.a.status = nullptr;
  p.logits_out = logits;
  p.rows = rows;
  p.V = V;
  p.d = d;
  p.n_split = lm_split_count(da->sms, rows, V);
  return lm_launch(false, *da, hidden, weight, p, (cudaStream_t)stream);
}

int eb_lmhead_reserve(eb_sampler_t* h, int32_t d) {
  if (!h || d < ebk::kLmBK || d % ebk::kLmBK != 0) return EB_ERR_INVALID_ARG;
  if (is_slice(h) || h->cfg.V % ebk::kLmBN != 0) return EB_ERR_UNSUPPORTED;
  if (h->lm_rec) return EB_OK;
  DeviceGuard guard(h->device);
  if (!guard.ok) return EB_ERR_CUDA;
  const int64_t rows = (int64_t)h->cfg.B * h->cfg.L;
  const int split = lm_split_count(h->sms, rows, h->cfg.V);
  void* ptr = nullptr;
  if (cudaMalloc(&ptr, (size_t)split * (size_t)rows * sizeof(ebk::SliceRecord)) != cudaSuccess) {
    cudaGetLastError();
    return EB_ERR_OUT_OF_MEMORY;
  }
  h->lm_rec = static_cast<ebk::SliceRecord*>(ptr);
  h->lm_split = split;
  return EB_OK;
}

int eb_lmhead_step(eb_sampler_t* h, const void* hidden, const void* weight, int32_t d, int step,
                   int32_t* canvas, uint8_t* committed, float* entropies, int32_t* argmax,
                   uint8_t* stop_flags, void* stream) {
  if (!h || !canvas || !committed || !entropies || !argmax || !stop_flags)
    return EB_ERR_INVALID_ARG;
  const eb_config_t& c = h->cfg;
  const int64_t rows = (int64_t)c.B * c.L;
  int rc = lm_check(hidden, weight, rows, c.V, d);
  if (rc != EB_OK) return rc;
  if (!h->lm_rec) return EB_ERR_INVALID_ARG;  // eb_lmhead_reserve first
  if (is_slice(h)) return EB_ERR_UNSUPPORTED;
  if (step < 0 || step >= c.num_steps) return EB_ERR_INVALID_ARG;
  if (step != 0 && step != h->last_step + 1) return EB_ERR_STEP_ORDER;
  DeviceGuard guard(h->device);
  if (!guard.ok) return EB_ERR_CUDA;
  DeviceAttrs* da = nullptr;
  if ((rc = device_attrs(h->device, &da)) != EB_OK) return rc;
  cudaStream_t st = (cudaStream_t)stream;

  // the fused contraction and sampler pass: one record per (position,
  // vocabulary range)
  ebk::LmArgs p;
  std::memset(&p, 0, sizeof(p));
  fill_args(h, p.a, step);
  p.a.committed = committed;
  p.a.stop_flags = stop_flags;
  p.rec = h->lm_rec;
  p.rows = (int)rows;
  p.V = c.V;
  p.d = d;
  p.n_split = h->lm_split;
  if ((rc = lm_launch(true, *da, hidden, weight, p, st)) != EB_OK) return rc;
  // the active canvases, then the records merged in vocabulary order and the
  // canvas decisions
  StepArgs a;
  fill_args(h, a, step);
  a.canvas = canvas;
  a.committed = committed;
  a.H_out = entropies;
  a.amax_out = argmax;
  a.stop_flags = stop_flags;
  ebk::active_index_kernel<<<1, 256, 0, st>>>(stop_flags, c.B, h->act_index);
  if (cudaGetLastError() != cudaSuccess) return EB_ERR_CUDA;
  const int32_t* act_index = h->act_index;
  const ebk::SliceRecord* rec = h->lm_rec;
  int n_slices = h->lm_split;
  void* cargs[] = {&a, &act_index, &rec, &n_slices};
  if (cudaLaunchKernel(h->combine.fn, dim3(h->combine.grid), dim3(ebk::kEpiThreads), cargs,
                       h->combine.smem, st) != cudaSuccess)
    return EB_ERR_CUDA;
  h->last_step = step;
  return EB_OK;
}

int eb_canvas_done(eb_sampler_t* h, const uint8_t* stop_flags, int b, int* done, void* stream) {
  if (!h || !stop_flags || !done) return EB_ERR_INVALID_ARG;
  if (b < -1 || b >= h->cfg.B) return EB_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok) return EB_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  const int n = h->cfg.B;
  uint8_t local[64];
  uint8_t* host = n <= 64 ? local : new (std::nothrow) uint8_t[n];
  if (!host) return EB_ERR_OUT_OF_MEMORY;
  uint32_t status = 0;
  int rc = EB_OK;
  if (cudaMemcpyAsync(host, stop_flags, (size_t)n, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(&status, h->status, sizeof(status), cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    rc = EB_ERR_CUDA;
  } else {
    int d = 1;
    if (b >= 0) {
      d = host[b] != 0;
    } else {
      for (int i = 0; i < n; ++i) d &= host[i] != 0;
    }
    *done = d;
    if (status != 0) rc = EB_ERR_DEVICE_STATUS;
  }
  if (host != local) delete[] host;
  return rc;
}

int eb_sampler_status(eb_sampler_t* h, uint32_t* status, int clear, void* stream) {
  if (!h || !status) return EB_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok) return EB_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(status, h->status, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return EB_ERR_CUDA;
  if (clear && cudaMemsetAsync(h->status, 0, sizeof(uint32_t), st) != cudaSuccess)
    return EB_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return EB_ERR_CUDA;
  return EB_OK;
}

int eb_sampler_draws(eb_sampler_t* h, int32_t* sample, float* pmax, void* stream) {
  if (!h) return EB_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok) return EB_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t BL = (size_t)h->cfg.B * (size_t)h->cfg.L;
  if (sample &&
      cudaMemcpyAsync(sample, h->sample, BL * sizeof(int32_t), cudaMemcpyDeviceToDevice, st) !=
          cudaSuccess)
    return EB_ERR_CUDA;
  if (pmax &&
      cudaMemcpyAsync(pmax, h->pmax, BL * sizeof(float), cudaMemcpyDeviceToDevice, st) !=
          cudaSuccess)
    return EB_ERR_CUDA;
  return EB_OK;
}

int eb_sampler_set_state(eb_sampler_t* h, const int32_t* prev_argmax, const int32_t* stable,
                         int next_step, void* stream) {
  if (!h || !prev_argmax) return EB_ERR_INVALID_ARG;
  if (next_step < 0 || next_step >= h->cfg.num_steps) return EB_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok) return EB_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t BL = (size_t)h->cfg.B * (size_t)h->cfg.L;
  if (cudaMemcpyAsync(h->prev_amax, prev_argmax, BL * sizeof(int32_t), cudaMemcpyDeviceToDevice,
                      st) != cudaSuccess)
    return EB_ERR_CUDA;
  if (stable) {
    if (cudaMemcpyAsync(h->stable, stable, (size_t)h->cfg.B * sizeof(int32_t),
                        cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return EB_ERR_CUDA;
  } else if (cudaMemsetAsync(h->stable, 0, (size_t)h->cfg.B * sizeof(int32_t), st) !=
             cudaSuccess) {
    return EB_ERR_CUDA;
  }
  h->last_step = next_step - 1;
  return EB_OK;
}

int eb_sampler_set_split_event(eb_sampler_t* h, void* event) {
  if (!h) return EB_ERR_INVALID_ARG;
  h->split_event = static_cast<cudaEvent_t>(event);
  return EB_OK;
}

int eb_sampler_set_wait_limit(eb_sampler_t* h, uint64_t limit_ns) {
  if (!h) return EB_ERR_INVALID_ARG;
  h->wait_ns = limit_ns == 0 ? ebk::kWaitLimitNs : limit_ns;
  return EB_OK;
}

size_t eb_sampler_workspace_bytes(const eb_sampler_t* h) { return h ? h->ws_bytes : 0; }

void eb_sampler_destroy(eb_sampler_t* h) {
  if (!h) return;
  {
    DeviceGuard guard(h->device);
    if (h->ws) cudaFree(h->ws);
    if (h->lm_rec) cudaFree(h->lm_rec);
  }
  delete h;
}

const char* eb_strerror(int code) {
  switch (code) {
    case EB_OK: return "ok";
    case EB_ERR_INVALID_ARG: return "invalid argument";
    case EB_ERR_CUDA: return "CUDA runtime error";
    case EB_ERR_OUT_OF_MEMORY: return "out of device memory";
    case EB_ERR_STEP_ORDER: return "step is neither 0 nor the previous step + 1";
    case EB_ERR_UNSUPPORTED: return "unsupported dtype or device";
    case EB_ERR_OVERFLOW: return "sizes exceed the library limits";
    case EB_ERR_DEVICE_STATUS: return "a kernel reported a problem (status word non-zero)";
    default: return "unknown status";
  }
}

int eb_version(void) { return 200; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free row statistics (eb_row_stats_noalloc)
//
// For callers that cannot or must not allocate device memory (a hard memory
// budget, a plugin given raw pointers, no sampler handle): the stream pass's
// records, row counters and per-row side outputs live in a static device
// array instead of a workspace.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocCtrlBytes = 256;  // stop flag, status, active index, count

}  // namespace

// Scratch: [0, 256) control words (the stop flag of the single pseudo-canvas
// and the status word must start at zero; the active index and count are
// written by the stream kernel), then the row records, the row counters
// (zero at the start of every call) and the per-row max probability and
// draw the stream kernel also writes.
static __device__ __align__(256) unsigned char g_noalloc_scratch[EB_NOALLOC_SCRATCH_BYTES];

namespace ebk {

// After the stream pass: if a wait of that pass gave up (status word set),
// every row's outputs are marked invalid rather than left stale.
__global__ void noalloc_mark_kernel(const uint32_t* status, float* H, int32_t* amax, int rows) {
  if (__ldcg(status) == 0u) return;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows; i += gridDim.x * blockDim.x) {
    H[i] = __int_as_float(0x7fc00000);
    amax[i] = -1;
  }
}

}  // namespace ebk

namespace {

struct NoAllocDevice {
  std::once_flag once;
  int rc = EB_ERR_CUDA;
  unsigned char* scratch = nullptr;
};
NoAllocDevice g_noalloc_dev[kMaxDevices];

// Once per device (the device current): the scratch's device address.
void noalloc_setup(NoAllocDevice& d) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
    cudaGetLastError();
    d.rc = EB_ERR_CUDA;
    return;
  }
  d.scratch = static_cast<unsigned char*>(p);
  d.rc = EB_OK;
}

template <int DT>
int noalloc_launch(const NoAllocDevice& nd, const DeviceAttrs& d, const void* logits, int32_t rows,
                   int32_t V, double T, float* entropies, int32_t* argmax, cudaStream_t st) {
  using Sh = ebk::StreamShape<DT>;
  const int ng = (int)(((int64_t)V + ebk::kGroup - 1) / ebk::kGroup);
  const uint64_t groups = (uint64_t)rows * (uint64_t)ng;
  const int grid = stream_grid<DT>(d.sms, groups);
  const int max_segs = row_max_segs(grid, (uint64_t)rows, ng);
  const uint64_t rec_bytes = (uint64_t)rows * (uint64_t)max_segs * (uint64_t)sizeof(Rec);
  const uint64_t side_bytes = (uint64_t)rows * 12u;  // counter, pmax, draw
  if (kNoAllocCtrlBytes + rec_bytes + side_bytes > EB_NOALLOC_SCRATCH_BYTES) return EB_ERR_OVERFLOW;
  if (ebk::stream_layout<DT>(1).total > d.optin) return EB_ERR_OVERFLOW;

  unsigned char* ctrl = nd.scratch;
  Rec* recs = reinterpret_cast<Rec*>(nd.scratch + kNoAllocCtrlBytes);
  int32_t* cnt = reinterpret_cast<int32_t*>(nd.scratch + kNoAllocCtrlBytes + rec_bytes);
  float* pmax = reinterpret_cast<float*>(cnt + rows);
  int32_t* sample = reinterpret_cast<int32_t*>(pmax + rows);
  if (cudaMemsetAsync(ctrl, 0, kNoAllocCtrlBytes, st) != cudaSuccess ||
      cudaMemsetAsync(cnt, 0, (size_t)rows * sizeof(int32_t), st) != cudaSuccess)
    return EB_ERR_CUDA;
  StepArgs a;
  std::memset(&a, 0, sizeof(a));
  a.logits = logits;
  a.H_out = entropies;
  a.amax_out = argmax;
  a.stop_flags = ctrl;  // one pseudo-canvas, active
  a.status = reinterpret_cast<uint32_t*>(ctrl + 4);
  a.act_index = reinterpret_cast<int32_t*>(ctrl + 8);
  a.n_act = reinterpret_cast<int32_t*>(ctrl + 12);
  a.recs = recs;
  a.row_cnt = cnt;
  a.pmax = pmax;
  a.sample = sample;
  a.wait_ns = ebk::kWaitLimitNs;
  a.B = 1;
  a.L = rows;  // the rows are the positions of one pseudo-canvas
  a.V = V;
  a.ng = ng;
  a.s = 0;
  a.N = 1;
  a.max_segs = max_segs;
  a.G1 = grid;
  const size_t elt = DT == ebk::kF32 ? 4 : 2;
  a.vec_ok = ((uintptr_t)logits % 16 == 0) && (((size_t)V * elt) % 16 == 0) ? 1 : 0;
  a.greedy = 1;  // no draw: the stream pass skips the Gumbel race
  a.c2 = (float)(1.4426950408889634 / T);
  a.iT = (float)(1.0 / T);
  a.V_tot = V;
  void* args[] = {&a};
  if (cudaLaunchKernel(reinterpret_cast<const void*>(&ebk::stream_kernel<DT>), dim3(grid),
                       dim3(Sh::kThreads), args, ebk::stream_layout<DT>(1).total, st) !=
      cudaSuccess)
    return EB_ERR_CUDA;
  ebk::noalloc_mark_kernel<<<std::min(64, (rows + 255) / 256), 256, 0, st>>>(a.status, entropies,
                                                                             argmax, rows);
  if (cudaGetLastError() != cudaSuccess) return EB_ERR_CUDA;
  return EB_OK;
}

}  // namespace

extern "C" int eb_row_stats_noalloc(const void* logits, int dtype, int32_t rows, int32_t V,
                                    double temperature, float* entropies, int32_t* argmax,
                                    void* stream) {
  if (!logits || !entropies || !argmax || rows < 1 || V < 1) return EB_ERR_INVALID_ARG;
  if (dtype != EB_F32 && dtype != EB_BF16) return EB_ERR_UNSUPPORTED;
  if (!(temperature > 0.0) || !std::isfinite(temperature)) return EB_ERR_INVALID_ARG;
  if ((uintptr_t)logits % (dtype == EB_F32 ? 4u : 2u) != 0) return EB_ERR_INVALID_ARG;
  if ((uint64_t)rows * (((uint64_t)V + ebk::kGroup - 1) / ebk::kGroup) >= (1ull << 46))
    return EB_ERR_OVERFLOW;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return EB_ERR_CUDA;
  DeviceAttrs* d = nullptr;
  int rc = device_attrs(device, &d);
  if (rc != EB_OK) return rc;
  NoAllocDevice& nd = g_noalloc_dev[device];
  std::call_once(nd.once, noalloc_setup, std::ref(nd));
  if (nd.rc != EB_OK) return nd.rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dtype == EB_F32
             ? noalloc_launch<ebk::kF32>(nd, *d, logits, rows, V, temperature, entropies, argmax,
                                         st)
             : noalloc_launch<ebk::kBF16>(nd, *d, logits, rows, V, temperature, entropies, argmax,
                                          st);
}
