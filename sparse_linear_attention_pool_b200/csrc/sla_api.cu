// C ABI of the library (declared in include/sla.h): argument validation,
// workspace layout and the launch sequence of the forward pass.
#include <math.h>

#include <vector>

#include "sla_internal.cuh"

using namespace sla;

namespace {

// Stage-timing record: SLA_NUM_STAGES + 1 events per recorded call.
struct StageTimer {
  std::vector<cudaEvent_t> events;
  int max_calls = 0;
  int used = 0;
};
StageTimer g_timer;

cudaEvent_t stage_event(int call, int k) { return g_timer.events[size_t(call) * (SLA_NUM_STAGES + 1) + k]; }

sla_status check_params(const sla_params* p) {
  if (p == nullptr) return SLA_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->N < 1) return SLA_ERR_INVALID_ARG;
  if (p->block_q != SLA_BLOCK || p->block_kv != SLA_BLOCK) return SLA_ERR_UNSUPPORTED;
  if (p->d != 64 && p->d != 128) return SLA_ERR_UNSUPPORTED;
  if (p->variant != SLA_VARIANT_SLA && p->variant != SLA_VARIANT_SLA2) return SLA_ERR_INVALID_ARG;
  if (p->precision != SLA_PREC_BF16 && p->precision != SLA_PREC_I8QK_F8PV)
    return SLA_ERR_INVALID_ARG;
  const long long Nb = (static_cast<long long>(p->N) + SLA_BLOCK - 1) / SLA_BLOCK;
  if (Nb > SLA_MAX_BLOCKS) return SLA_ERR_UNSUPPORTED;
  if (static_cast<long long>(p->B) * p->H > 65535) return SLA_ERR_UNSUPPORTED;  // grid.y limit
  if (p->k_crit < 1 || p->k_crit > Nb || p->k_neg < 0 || p->k_crit + p->k_neg > Nb)
    return SLA_ERR_INVALID_ARG;
  if (!(p->softmax_scale >= 0.0f) || isinf(p->softmax_scale)) return SLA_ERR_INVALID_ARG;
  if (p->variant == SLA_VARIANT_SLA2) {
    if (p->alpha == nullptr) return SLA_ERR_INVALID_ARG;
    if ((p->proj_q == nullptr) != (p->proj_k == nullptr)) return SLA_ERR_INVALID_ARG;
  }
  if (p->precision == SLA_PREC_I8QK_F8PV && p->d != 128) return SLA_ERR_UNSUPPORTED;
  if (p->phi != SLA_PHI_SOFTMAX && p->phi != SLA_PHI_ELU1) return SLA_ERR_INVALID_ARG;
  return SLA_OK;
}

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

}  // namespace

extern "C" {

int sla_abi_version(void) { return SLA_ABI_VERSION; }

const char* sla_status_string(sla_status status) {
  switch (status) {
    case SLA_OK: return "ok";
    case SLA_ERR_INVALID_ARG: return "invalid argument";
    case SLA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SLA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SLA_ERR_ALIGNMENT: return "tensor address not 16-byte aligned";
    case SLA_ERR_CUDA: return "CUDA error";
    case SLA_ERR_DEVICE_TIMEOUT: return "bounded device wait expired";
    case SLA_ERR_DEVICE_CHECK: return "in-kernel consistency check failed";
  }
  return "unknown status";
}

sla_status sla_validate(const sla_params* p) { return check_params(p); }

size_t sla_workspace_size(const sla_params* p) {
  if (check_params(p) != SLA_OK) return 0;
  return make_layout(*p).total;
}

}  // extern "C"

namespace {

sla_status run_forward(const void* Q, const void* K, const void* V, void* O, const sla_params* p,
                       void* workspace, size_t workspace_bytes, void* stream, const sla_saved* saved) {
  sla_status st = check_params(p);
  if (st != SLA_OK) return st;
  if (!Q || !K || !V || !O) return SLA_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16))
    return SLA_ERR_ALIGNMENT;
  if ((p->w_proj && !aligned(p->w_proj, 16)) || (p->proj_q && !aligned(p->proj_q, 16)) ||
      (p->proj_k && !aligned(p->proj_k, 16)) || (p->alpha && !aligned(p->alpha, 4)))
    return SLA_ERR_ALIGNMENT;
  const Layout L = make_layout(*p);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < L.total)
    return SLA_ERR_WORKSPACE;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  auto bf = [](const void* x) { return static_cast<const __nv_bfloat16*>(x); };
  float* qbar = reinterpret_cast<float*>(ws + L.qbar);
  float* kbar = reinterpret_cast<float*>(ws + L.kbar);
  float* scores = reinterpret_cast<float*>(ws + L.scores);
  int8_t* mc = reinterpret_cast<int8_t*>(ws + L.mc);
  int32_t* crit = reinterpret_cast<int32_t*>(ws + L.crit);
  int32_t* neg = reinterpret_cast<int32_t*>(ws + L.neg);
  __nv_bfloat16* phik = reinterpret_cast<__nv_bfloat16*>(ws + L.phik);
  float* zblk = reinterpret_cast<float*>(ws + L.zblk);
  float* hpart = reinterpret_cast<float*>(ws + L.hpart);
  float* zpart = reinterpret_cast<float*>(ws + L.zpart);
  float* htot32 = reinterpret_cast<float*>(ws + L.htot32);
  __nv_bfloat16* htot16 = reinterpret_cast<__nv_bfloat16*>(ws + L.htot16);
  float* ztot = reinterpret_cast<float*>(ws + L.ztot);
  __nv_bfloat16* phiq = L.pre ? reinterpret_cast<__nv_bfloat16*>(ws + L.phiq) : nullptr;
  float* zi = L.pre ? reinterpret_cast<float*>(ws + L.zi) : nullptr;
  int8_t* qcode = L.quant ? reinterpret_cast<int8_t*>(ws + L.qcode) : nullptr;
  int8_t* kcode = L.quant ? reinterpret_cast<int8_t*>(ws + L.kcode) : nullptr;
  uint8_t* vcode = L.quant ? reinterpret_cast<uint8_t*>(ws + L.vcode) : nullptr;
  float* qscale = L.quant ? reinterpret_cast<float*>(ws + L.qscale) : nullptr;
  float* kscale = L.quant ? reinterpret_cast<float*>(ws + L.kscale) : nullptr;
  float* vscale = L.quant ? reinterpret_cast<float*>(ws + L.vscale) : nullptr;
  const bool sla2 = p->variant == SLA_VARIANT_SLA2;
  const int elu1 = p->phi == SLA_PHI_ELU1 ? 1 : 0;

  const int call = g_timer.used < g_timer.max_calls ? g_timer.used++ : -1;
  auto mark = [&](int k) {
    if (call >= 0) cudaEventRecord(stage_event(call, k), s);
  };
  int* status = reinterpret_cast<int*>(ws + L.status);
  const __nv_bfloat16* proj_q = sla2 ? bf(p->proj_q) : nullptr;
  const __nv_bfloat16* proj_k = sla2 ? bf(p->proj_k) : nullptr;
  cudaError_t e = cudaMemsetAsync(ws + L.status, 0, 256, s);
  // stages: 0 Q side (pooling; phi(Q) when precomputed; the general path pools
  // K here too), 1 K / V side (phi(K), z_j, partial H and Z), 2 scores,
  // 3 classification, 4 H_tot / Z_tot (and Z_i), 5 attention
  mark(0);
  if (L.stream) {
    if (e == cudaSuccess) e = launch_q_stream(L, bf(Q), proj_q, qbar, phiq, elu1, status, s);
    mark(1);
    if (e == cudaSuccess)
      e = launch_kv_stream(L, bf(K), bf(V), proj_k, kbar, phik, zblk, hpart, zpart, elu1, status, s);
  } else {
    if (e == cudaSuccess)
      e = launch_pool(L, bf(Q), bf(K), proj_q, proj_k, qbar, kbar, qcode, kcode, qscale, kscale, phiq, elu1, s);
    mark(1);
    if (e == cudaSuccess) e = launch_phik_hz(L, bf(K), bf(V), phik, zblk, hpart, zpart, vcode, vscale, elu1, s);
  }
  mark(2);
  if (e == cudaSuccess) e = launch_scores(L, qbar, kbar, scores, s);
  mark(3);
  if (e == cudaSuccess) e = launch_classify(L, scores, mc, crit, neg, s);
  mark(4);
  if (e == cudaSuccess) e = launch_hz_reduce(L, zpart, hpart, htot32, htot16, ztot, s);
  if (e == cudaSuccess && L.pre)
    e = launch_zi(L, crit, neg, zblk, ztot, zi, status, s);
  mark(5);
  if (e == cudaSuccess) {
    AttnArgs a{};
    a.Q = bf(Q);
    a.K = bf(K);
    a.V = bf(V);
    a.O = static_cast<__nv_bfloat16*>(O);
    a.phik = phik;
    a.crit = crit;
    a.neg = neg;
    a.htot32 = htot32;
    a.htot16 = htot16;
    a.phiq = phiq;
    a.zi = zi;
    a.ztot = ztot;
    a.zblk = zblk;
    a.phi_elu1 = elu1;
    a.w_proj = sla2 ? nullptr : bf(p->w_proj);
    a.alpha = sla2 ? p->alpha : nullptr;
    a.status = reinterpret_cast<int*>(ws + L.status);
    a.qcode = qcode;
    a.kcode = kcode;
    a.vcode = vcode;
    a.qscale = qscale;
    a.kscale = kscale;
    a.vscale = vscale;
    a.H = p->H;
    a.N = p->N;
    a.Nb = L.Nb;
    a.kc = L.kc;
    a.kn = L.kn;
    const float scale = p->softmax_scale > 0.0f ? p->softmax_scale : 1.0f / sqrtf(float(p->d));
    a.scale_log2 = scale * 1.4426950408889634f;
    if (saved != nullptr) {
      a.save_os = static_cast<__nv_bfloat16*>(saved->o_s);
      a.save_ol = static_cast<__nv_bfloat16*>(saved->o_l);
      a.save_lse = saved->lse;
      a.save_den = saved->den;
    }
    e = launch_attention(a, L.BH, L.d, sla2 ? kModeSLA2 : kModeSLA, s);
  }
  mark(6);
  return e == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}

bool saved_ok(const sla_saved* sv) {
  return sv != nullptr && sv->o_s && sv->o_l && sv->lse && sv->den && aligned(sv->o_s, 16) && aligned(sv->o_l, 16) &&
         aligned(sv->lse, 4) && aligned(sv->den, 4);
}

}  // namespace

extern "C" {

sla_status sla_forward(const void* Q, const void* K, const void* V, void* O, const sla_params* p,
                       void* workspace, size_t workspace_bytes, void* stream) {
  return run_forward(Q, K, V, O, p, workspace, workspace_bytes, stream, nullptr);
}

sla_status sla_forward_train(const void* Q, const void* K, const void* V, void* O, const sla_params* p,
                             const sla_saved* saved, void* workspace, size_t workspace_bytes, void* stream) {
  sla_status st = check_params(p);
  if (st != SLA_OK) return st;
  if (p->precision != SLA_PREC_BF16) return SLA_ERR_UNSUPPORTED;
  if (saved == nullptr || !saved->o_s || !saved->o_l || !saved->lse || !saved->den) return SLA_ERR_INVALID_ARG;
  if (!saved_ok(saved)) return SLA_ERR_ALIGNMENT;
  return run_forward(Q, K, V, O, p, workspace, workspace_bytes, stream, saved);
}

size_t sla_backward_workspace_size(const sla_params* p) {
  if (check_params(p) != SLA_OK) return 0;
  return make_bw_layout(*p).total;
}

sla_status sla_backward(const void* Q, const void* K, const void* V, const void* dO, const sla_params* p,
                        const sla_saved* saved, const void* fwd_workspace, size_t fwd_workspace_bytes, void* dQ,
                        void* dK, void* dV, float* dW, float* dalpha, void* workspace, size_t workspace_bytes,
                        void* stream) {
  sla_status st = check_params(p);
  if (st != SLA_OK) return st;
  if (p->precision != SLA_PREC_BF16) return SLA_ERR_UNSUPPORTED;
  const bool sla2 = p->variant == SLA_VARIANT_SLA2;
  if (!Q || !K || !V || !dO || !dQ || !dK || !dV || saved == nullptr) return SLA_ERR_INVALID_ARG;
  if (!saved->o_s || !saved->o_l || !saved->lse || !saved->den) return SLA_ERR_INVALID_ARG;
  if ((dW != nullptr && sla2) || (dalpha != nullptr && !sla2)) return SLA_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(dO, 16) || !aligned(dQ, 16) ||
      !aligned(dK, 16) || !aligned(dV, 16) || !saved_ok(saved) || (dW && !aligned(dW, 4)) ||
      (dalpha && !aligned(dalpha, 4)) || (p->w_proj && !aligned(p->w_proj, 16)))
    return SLA_ERR_ALIGNMENT;
  const Layout L = make_layout(*p);
  const BwLayout BL = make_bw_layout(*p);
  if (fwd_workspace == nullptr || !aligned(fwd_workspace, 256) || fwd_workspace_bytes < L.total)
    return SLA_ERR_WORKSPACE;
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < BL.total) return SLA_ERR_WORKSPACE;
  const unsigned char* fw = static_cast<const unsigned char*>(fwd_workspace);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  auto bf = [](const void* x) { return static_cast<const __nv_bfloat16*>(x); };
  BwdArgs a{};
  a.L = BL;
  a.Q = bf(Q);
  a.K = bf(K);
  a.V = bf(V);
  a.dO = bf(dO);
  a.save_os = bf(saved->o_s);
  a.save_ol = bf(saved->o_l);
  a.save_lse = saved->lse;
  a.save_den = saved->den;
  a.w_proj = sla2 ? nullptr : bf(p->w_proj);
  a.alpha = sla2 ? p->alpha : nullptr;
  a.phik = reinterpret_cast<const __nv_bfloat16*>(fw + L.phik);
  a.htot = reinterpret_cast<const float*>(fw + L.htot32);
  a.ztot = reinterpret_cast<const float*>(fw + L.ztot);
  a.zblk = reinterpret_cast<const float*>(fw + L.zblk);
  a.mc = reinterpret_cast<const int8_t*>(fw + L.mc);
  a.crit = reinterpret_cast<const int32_t*>(fw + L.crit);
  a.neg = reinterpret_cast<const int32_t*>(fw + L.neg);
  a.dnum = reinterpret_cast<__nv_bfloat16*>(ws + BL.dnum);
  a.phiq = reinterpret_cast<__nv_bfloat16*>(ws + BL.phiq);
  a.Drow = reinterpret_cast<float*>(ws + BL.drow);
  a.dden = reinterpret_cast<float*>(ws + BL.dden);
  a.dzblk = reinterpret_cast<float*>(ws + BL.dzblk);
  a.dztot = reinterpret_cast<float*>(ws + BL.dztot);
  a.hblk = reinterpret_cast<__nv_bfloat16*>(ws + BL.hblk);
  a.dhblk = reinterpret_cast<__nv_bfloat16*>(ws + BL.dhblk);
  a.dhtot = reinterpret_cast<float*>(ws + BL.dhtot);
  a.dwpart = reinterpret_cast<float*>(ws + BL.dwpart);
  a.dapart = reinterpret_cast<float*>(ws + BL.dapart);
  a.colC = reinterpret_cast<int*>(ws + BL.colc);
  a.colE = reinterpret_cast<int*>(ws + BL.cole);
  a.cntC = reinterpret_cast<int*>(ws + BL.cntc);
  a.cntE = reinterpret_cast<int*>(ws + BL.cnte);
  a.dks = BL.d == 128 ? reinterpret_cast<float*>(ws + BL.dks) : nullptr;
  a.dvs = BL.d == 128 ? reinterpret_cast<float*>(ws + BL.dvs) : nullptr;
  a.dqs = BL.d == 128 ? reinterpret_cast<float*>(ws + BL.dqs) : nullptr;
  a.status = reinterpret_cast<int*>(const_cast<unsigned char*>(fw) + L.status);
  a.dQ = static_cast<__nv_bfloat16*>(dQ);
  a.dK = static_cast<__nv_bfloat16*>(dK);
  a.dV = static_cast<__nv_bfloat16*>(dV);
  a.dW = sla2 ? nullptr : dW;
  a.dalpha = sla2 ? dalpha : nullptr;
  a.scale = p->softmax_scale > 0.0f ? p->softmax_scale : 1.0f / sqrtf(float(p->d));
  a.sla = !sla2;
  a.phi_elu1 = p->phi == SLA_PHI_ELU1 ? 1 : 0;
  const cudaError_t e = launch_backward(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}

sla_status sla_router_soft_topk(const void* Q, const void* K, const sla_params* p, float tau,
                                float* m_soft, float* lambda, float* pc, void* workspace,
                                size_t workspace_bytes, void* stream) {
  sla_status st = check_params(p);
  if (st != SLA_OK) return st;
  if (!Q || !K || !m_soft) return SLA_ERR_INVALID_ARG;
  if (!(tau > 0.0f) || isinf(tau) || isinf(1.4426950408889634f / tau)) return SLA_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(m_soft, 4) || (lambda && !aligned(lambda, 4)) ||
      (pc && !aligned(pc, 4)))
    return SLA_ERR_ALIGNMENT;
  if ((p->proj_q && !aligned(p->proj_q, 16)) || (p->proj_k && !aligned(p->proj_k, 16)))
    return SLA_ERR_ALIGNMENT;
  const Layout L = make_layout(*p);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < L.total)
    return SLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  auto bf = [](const void* x) { return static_cast<const __nv_bfloat16*>(x); };
  float* qbar = reinterpret_cast<float*>(ws + L.qbar);
  float* kbar = reinterpret_cast<float*>(ws + L.kbar);
  float* scores = reinterpret_cast<float*>(ws + L.scores);
  const bool sla2 = p->variant == SLA_VARIANT_SLA2;
  cudaError_t e = launch_pool(L, bf(Q), bf(K), sla2 ? bf(p->proj_q) : nullptr, sla2 ? bf(p->proj_k) : nullptr,
                              qbar, kbar, nullptr, nullptr, nullptr, nullptr, nullptr, 0, s);
  if (e == cudaSuccess) e = launch_scores(L, qbar, kbar, scores, s);
  const float scale = p->softmax_scale > 0.0f ? p->softmax_scale : 1.0f / sqrtf(float(p->d));
  if (e == cudaSuccess) e = launch_soft_topk(L, scores, m_soft, lambda, pc, scale, tau, s);
  return e == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}

sla_status sla_stage_timing(int max_calls) {
  if (max_calls < 0) return SLA_ERR_INVALID_ARG;
  for (cudaEvent_t ev : g_timer.events) cudaEventDestroy(ev);
  g_timer = StageTimer{};
  const size_t n = size_t(max_calls) * (SLA_NUM_STAGES + 1);
  g_timer.events.reserve(n);
  for (size_t i = 0; i < n; ++i) {
    cudaEvent_t ev;
    if (cudaEventCreate(&ev) != cudaSuccess) {
      sla_stage_timing(0);
      return SLA_ERR_CUDA;
    }
    g_timer.events.push_back(ev);
  }
  g_timer.max_calls = max_calls;
  return SLA_OK;
}

sla_status sla_stage_times(float* ms, int* calls) {
  if (ms == nullptr || calls == nullptr) return SLA_ERR_INVALID_ARG;
  for (int k = 0; k < SLA_NUM_STAGES; ++k) ms[k] = 0.0f;
  *calls = g_timer.used;
  for (int c = 0; c < g_timer.used; ++c) {
    if (cudaEventSynchronize(stage_event(c, SLA_NUM_STAGES)) != cudaSuccess) return SLA_ERR_CUDA;
    for (int k = 0; k < SLA_NUM_STAGES; ++k) {
      float t = 0.0f;
      if (cudaEventElapsedTime(&t, stage_event(c, k), stage_event(c, k + 1)) != cudaSuccess)
        return SLA_ERR_CUDA;
      ms[k] += t;
    }
  }
  g_timer.used = 0;
  return SLA_OK;
}

sla_status sla_get_mask(const sla_params* p, const void* workspace, int8_t* mc, int32_t* crit,
                        int32_t* neg, void* stream) {
  sla_status st = check_params(p);
  if (st != SLA_OK) return st;
  if (workspace == nullptr || !aligned(workspace, 256)) return SLA_ERR_WORKSPACE;
  const Layout L = make_layout(*p);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned char* ws = static_cast<const unsigned char*>(workspace);
  const size_t rows = size_t(L.BH) * L.Nb;
  cudaError_t e = cudaSuccess;
  if (mc) e = cudaMemcpyAsync(mc, ws + L.mc, rows * L.Nb, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && crit)
    e = cudaMemcpyAsync(crit, ws + L.crit, rows * L.kc * 4, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && neg && L.kn > 0)
    e = cudaMemcpyAsync(neg, ws + L.neg, rows * L.kn * 4, cudaMemcpyDeviceToDevice, s);
  return e == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}

sla_status sla_get_pooled(const sla_params* p, const void* workspace, float* qbar, float* kbar,
                          void* stream) {
  sla_status st = check_params(p);
  if (st != SLA_OK) return st;
  if (workspace == nullptr || !aligned(workspace, 256)) return SLA_ERR_WORKSPACE;
  const Layout L = make_layout(*p);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned char* ws = static_cast<const unsigned char*>(workspace);
  const size_t bytes = size_t(L.BH) * L.Nb * L.d * 4;
  cudaError_t e = cudaSuccess;
  if (qbar) e = cudaMemcpyAsync(qbar, ws + L.qbar, bytes, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && kbar)
    e = cudaMemcpyAsync(kbar, ws + L.kbar, bytes, cudaMemcpyDeviceToDevice, s);
  return e == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}

sla_status sla_get_quantized(const sla_params* p, const void* workspace, int8_t* qcode, int8_t* kcode,
                             uint8_t* vcode, float* qscale, float* kscale, float* vscale, void* stream) {
  sla_status st = check_params(p);
  if (st != SLA_OK) return st;
  if (p->precision != SLA_PREC_I8QK_F8PV) return SLA_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned(workspace, 256)) return SLA_ERR_WORKSPACE;
  const Layout L = make_layout(*p);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned char* ws = static_cast<const unsigned char*>(workspace);
  const size_t cbytes = size_t(L.BH) * L.Npad * L.d, sbytes = size_t(L.BH) * L.Nb * 4;
  cudaError_t e = cudaSuccess;
  auto cp = [&](void* dst, size_t off, size_t n) {
    if (dst && e == cudaSuccess) e = cudaMemcpyAsync(dst, ws + off, n, cudaMemcpyDeviceToDevice, s);
  };
  cp(qcode, L.qcode, cbytes);
  cp(kcode, L.kcode, cbytes);
  cp(vcode, L.vcode, cbytes);
  cp(qscale, L.qscale, sbytes);
  cp(kscale, L.kscale, sbytes);
  cp(vscale, L.vscale, sbytes);
  return e == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}

sla_status sla_read_device_status(const void* workspace, void* stream) {
  if (workspace == nullptr) {  // the no-alloc entry point's static workspace on this device
    void* ws = nullptr;
    const sla_status st = noalloc_workspace_address(&ws);
    if (st != SLA_OK) return st;
    workspace = ws;
  }
  if (!aligned(workspace, 256)) return SLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return SLA_ERR_CUDA;
  if (word == kDevOk) return SLA_OK;
  return word == kDevTimeout ? SLA_ERR_DEVICE_TIMEOUT : SLA_ERR_DEVICE_CHECK;
}

sla_status sla_dense_forward(const void* Q, const void* K, const void* V, void* O, int B, int H,
                             int N, int d, float softmax_scale, void* stream) {
  if (!Q || !K || !V || !O || B < 1 || H < 1 || N < 1) return SLA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SLA_ERR_UNSUPPORTED;
  if (!(softmax_scale >= 0.0f) || isinf(softmax_scale)) return SLA_ERR_INVALID_ARG;
  const long long Nb = (static_cast<long long>(N) + SLA_BLOCK - 1) / SLA_BLOCK;
  if (Nb > SLA_MAX_BLOCKS || static_cast<long long>(B) * H > 65535) return SLA_ERR_UNSUPPORTED;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16))
    return SLA_ERR_ALIGNMENT;
  AttnArgs a{};
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.K = static_cast<const __nv_bfloat16*>(K);
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.O = static_cast<__nv_bfloat16*>(O);
  a.H = H;
  a.N = N;
  a.Nb = int(Nb);
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / sqrtf(float(d));
  a.scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e = launch_attention(a, B * H, d, kModeDense, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}

}  // extern "C"
