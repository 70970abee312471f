// SoftTop-k router forward: the differentiable stand-in for the hard Top-k in
// the first training stage of SLA2's router (SLA2 article, mcffsbgs.com,
// two-stage training paragraphs: a sigmoid with a temperature instead of the
// Top-k selection; "SLA2 -- L3 Cross-Paper Synthesis", section 3: lambda_i per
// row by binary search so that the row meets its sum constraint).
//
// Per row i of the pooled scores s (the float32 scores of the mask stage):
//   Pc_ij = softmax_j(scale s_ij)                  (SLA structured summary, formula 1)
//   M_ij  = sigmoid((Pc_ij - lambda_i) / tau),     sum_j M_ij = k
// The row sum falls strictly in lambda; the root is bracketed by
// [min Pc - tau logit(k/n), max Pc - tau logit(k/n)] (every term is then >= or
// <= k/n) and found by bracketed Newton steps that fall back to bisection. The
// residual sum_j M_ij - k is accumulated as (#{Pc_ij > lambda} - k) plus the
// signed sigmoid tails t = sigmoid(-|x|), each small and accurate, so lambda
// stays determined when the sigmoids of a row saturate at 0 and 1.
//
// One warp per row, the row's Nb values in registers (VPL per lane). Every lane
// holds the same bracket (the xor-butterfly sums are bitwise identical across
// lanes), so the loop exit is warp-uniform. Bound: the MUFU unit, two
// operations (2^x, reciprocal) per element per step.
#include "sla_internal.cuh"

namespace sla {
namespace {

constexpr int kRouterWarps = 8;
constexpr int kMaxSteps = 160;  // steps per row; fp32 brackets collapse well before this
// Stop once |sum_j M_ij - k| <= kResidStop: moving lambda to the exact root
// would change each M_ij by at most the residual (dM_j = t_j (1 - t_j)
// dlambda / tau with dlambda = r tau / sum_j t_j (1 - t_j)).
constexpr float kResidStop = 5e-6f;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// the smaller of sigmoid(x) and 1 - sigmoid(x), x given in log2 units (x log2 e)
__device__ __forceinline__ float sigmoid_tail(float x2) {
  const float e = ex2_approx(-fabsf(x2));
  return __fdividef(e, 1.0f + e);
}

template <int VPL>
__global__ void __launch_bounds__(32 * kRouterWarps) soft_topk_kernel(
    const float* __restrict__ S, float* __restrict__ M, float* __restrict__ lambda,
    float* __restrict__ pc_out, int Nb, int rows, int k, float scale_log2, float inv_tau_log2,
    float tau, float off) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kRouterWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float* srow = S + size_t(row) * Nb;

  // Pc = softmax(scale s) over the row
  float p[VPL];
  float mx = -INFINITY;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int j = lane + 32 * v;
    p[v] = j < Nb ? srow[j] * scale_log2 : -INFINITY;
    mx = fmaxf(mx, p[v]);
  }
  mx = warp_max(mx);
  float sum = 0.0f;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int j = lane + 32 * v;
    p[v] = j < Nb ? ex2_approx(p[v] - mx) : 0.0f;
    sum += p[v];
  }
  sum = warp_sum(sum);
  float pmin = INFINITY, pmax = -INFINITY;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int j = lane + 32 * v;
    if (j < Nb) {
      p[v] = p[v] / sum;
      pmin = fminf(pmin, p[v]);
      pmax = fmaxf(pmax, p[v]);
      if (pc_out) pc_out[size_t(row) * Nb + j] = p[v];
    }
  }
  pmin = warp_min(pmin);
  pmax = warp_max(pmax);

  float* mrow = M + size_t(row) * Nb;
  if (k >= Nb) {  // every block selected: M = 1, lambda = -inf
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int j = lane + 32 * v;
      if (j < Nb) mrow[j] = 1.0f;
    }
    if (lambda && lane == 0) lambda[row] = -INFINITY;
    return;
  }

  // Bracketed Newton: each step evaluates the residual r and the slope
  // sum_j t_j (1 - t_j) = -tau f'(lambda) at lam, narrows the bracket by the
  // sign of r, and moves to the Newton point when it falls strictly inside the
  // bracket, else to the bracket's midpoint (plain bisection). The root is
  // unique, so this reaches the root bisection alone would, in 6-13 steps
  // instead of 21-32 on the router's score rows.
  float lo = pmin - off, hi = pmax - off;
  float lam = 0.5f * (lo + hi);
  for (int it = 0; it < kMaxSteps; ++it) {
    int above = 0;
    float tail = 0.0f, slope = 0.0f;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int j = lane + 32 * v;
      if (j < Nb) {
        const float x2 = (p[v] - lam) * inv_tau_log2;
        const float t = sigmoid_tail(x2);
        const bool pos = x2 > 0.0f;
        above += pos;
        tail += pos ? -t : t;
        slope = fmaf(t, 1.0f - t, slope);
      }
    }
    above = warp_sum_i(above);
    tail = warp_sum(tail);
    slope = warp_sum(slope);
    const float resid = float(above - k) + tail;  // sum_j M_ij - k at lam
    if (fabsf(resid) <= kResidStop) break;
    if (resid > 0.0f)
      lo = lam;  // the root lies right of lam
    else
      hi = lam;
    const float mid = 0.5f * (lo + hi);
    if (!(mid > lo && mid < hi)) break;  // no float left strictly inside the bracket
    const float nl = lam + resid * tau / slope;
    const float next = (nl > lo && nl < hi) ? nl : mid;
    if (next == lam) break;
    lam = next;
  }
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int j = lane + 32 * v;
    if (j < Nb) {
      const float x2 = (p[v] - lam) * inv_tau_log2;
      const float t = sigmoid_tail(x2);
      mrow[j] = x2 > 0.0f ? 1.0f - t : t;
    }
  }
  if (lambda && lane == 0) lambda[row] = lam;
}

template <int VPL>
cudaError_t launch_vpl(const Layout& L, const float* scores, float* m, float* lambda, float* pc,
                       float scale, float tau, double off, cudaStream_t s) {
  const int rows = L.BH * L.Nb;
  soft_topk_kernel<VPL><<<(rows + kRouterWarps - 1) / kRouterWarps, 32 * kRouterWarps, 0, s>>>(
      scores, m, lambda, pc, L.Nb, rows, L.kc, scale * kLog2e, kLog2e / tau, tau, float(off));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_soft_topk(const Layout& L, const float* scores, float* m, float* lambda, float* pc,
                             float scale, float tau, cudaStream_t s) {
  // bracket offset tau logit(k / Nb), unused when k = Nb
  const double off = L.kc < L.Nb ? double(tau) * log(double(L.kc) / double(L.Nb - L.kc)) : 0.0;
  if (L.Nb <= 256) return launch_vpl<8>(L, scores, m, lambda, pc, scale, tau, off, s);
  if (L.Nb <= 512) return launch_vpl<16>(L, scores, m, lambda, pc, scale, tau, off, s);
  if (L.Nb <= 1024) return launch_vpl<32>(L, scores, m, lambda, pc, scale, tau, off, s);
  if (L.Nb <= 1280) return launch_vpl<40>(L, scores, m, lambda, pc, scale, tau, off, s);
  if (L.Nb <= 1536) return launch_vpl<48>(L, scores, m, lambda, pc, scale, tau, off, s);
  if (L.Nb <= 2048) return launch_vpl<64>(L, scores, m, lambda, pc, scale, tau, off, s);
  return launch_vpl<128>(L, scores, m, lambda, pc, scale, tau, off, s);
}

}  // namespace sla
