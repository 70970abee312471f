// Attention-weight prediction and block classification (steps 1-2 of the
// forward): block mean pooling of Q and K, SLA2's router projections, the
// pooled scores s_ij = qbar_i . kbar_j and the per-row three-way split into
// critical / marginal / negligible blocks (the compressed mask Mc).
//
// Source: SLA structured summary (aipaper.cc), section 4 "Methodology",
// formula 1 (Pc = softmax(pool(Q) pool(K)^T / sqrt(d)), pool = mean over the
// sequence dimension) and formula 2 (Mc = 1 for the top kh % of a row, -1 for
// the bottom kl %, 0 otherwise); router: SLA2 notes (zhaifeiyue.github.io)
// section 2 and SLA2 article (mcffsbgs.com), two learnable projection
// matrices applied to Q and K before pooling.
//
// Arithmetic is fixed so that the mask is reproducible bit for bit: every
// sum runs in float32 in ascending index order, starting from +0, with the
// products and sums rounded separately (__fmul_rn / __fadd_rn are never
// contracted into FMA). Softmax and the 1/sqrt(d) scale are increasing, so
// the ranking uses the raw scores. Ties rank by ascending block index.
#include "sla_internal.cuh"

namespace sla {

// ---------------------------------------------------------------------------
// pooling (+ router)
// ---------------------------------------------------------------------------
// CTA: 128 threads = (128 / (d/8)) blocks x (d/8) threads; a thread owns 8
// adjacent columns of one 64-token block. grid = (ceil(Nb / bpc), BH, 2).
template <int D>
__global__ void __launch_bounds__(128) pool_kernel(const __nv_bfloat16* __restrict__ Q,
                                                   const __nv_bfloat16* __restrict__ K,
                                                   const __nv_bfloat16* __restrict__ proj_q,
                                                   const __nv_bfloat16* __restrict__ proj_k,
                                                   float* __restrict__ qbar, float* __restrict__ kbar,
                                                   int N, int Npad, int Nb) {
  constexpr int TPB = D / 8;        // threads per block row
  constexpr int BPC = 128 / TPB;    // blocks per CTA
  __shared__ float pooled[BPC][D];
  const int which = blockIdx.z;     // 0: Q, 1: K
  const int bh = blockIdx.y;
  const int lb = threadIdx.x / TPB;
  const int c0 = (threadIdx.x % TPB) * 8;
  const int blk = blockIdx.x * BPC + lb;
  const __nv_bfloat16* X = which == 0 ? Q : K;
  const __nv_bfloat16* Wp = which == 0 ? proj_q : proj_k;
  float* out = which == 0 ? qbar : kbar;

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  const bool live = blk < Nb;
  if (live) {
    const int n = min(kBlock, N - blk * kBlock);
    const __nv_bfloat16* base = X + (size_t(bh) * Npad + size_t(blk) * kBlock) * D + c0;
#pragma unroll 8
    for (int t = 0; t < n; ++t) {
      uint4 raw = *reinterpret_cast<const uint4*>(base + size_t(t) * D);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] = __fadd_rn(acc[2 * e], bf16_lo(w[e]));
        acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], bf16_hi(w[e]));
      }
    }
    if (n == kBlock) {
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = __fmul_rn(acc[e], 0.015625f);
    } else {
      const float fn = float(n);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = __fdiv_rn(acc[e], fn);
    }
  }
  if (Wp != nullptr) {  // router: out[c] = sum_k pooled[k] * W[k][c], k ascending
#pragma unroll
    for (int e = 0; e < 8; ++e) pooled[lb][c0 + e] = acc[e];
    __syncthreads();
    float r[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) r[e] = 0.0f;
    for (int k = 0; k < D; ++k) {
      const float x = pooled[lb][k];
      uint4 raw = *reinterpret_cast<const uint4*>(Wp + size_t(k) * D + c0);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        r[2 * e] = __fadd_rn(r[2 * e], __fmul_rn(x, bf16_lo(w[e])));
        r[2 * e + 1] = __fadd_rn(r[2 * e + 1], __fmul_rn(x, bf16_hi(w[e])));
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = r[e];
  }
  if (live) {
    float4* o = reinterpret_cast<float4*>(out + (size_t(bh) * Nb + blk) * D + c0);
    o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

cudaError_t launch_pool(const Layout& L, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                        const __nv_bfloat16* proj_q, const __nv_bfloat16* proj_k, float* qbar,
                        float* kbar, cudaStream_t s) {
  const int bpc = 128 / (L.d / 8);
  dim3 grid((L.Nb + bpc - 1) / bpc, L.BH, 2);
  if (L.d == 128)
    pool_kernel<128><<<grid, 128, 0, s>>>(Q, K, proj_q, proj_k, qbar, kbar, L.N, L.Npad, L.Nb);
  else
    pool_kernel<64><<<grid, 128, 0, s>>>(Q, K, proj_q, proj_k, qbar, kbar, L.N, L.Npad, L.Nb);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// pooled scores
// ---------------------------------------------------------------------------
// CTA: 16 x 16 threads, a 64 x 64 tile of S; thread (tx, ty) owns rows
// ty + 16a and columns tx + 16b. k runs ascending across 32-wide chunks.
__global__ void __launch_bounds__(256) scores_kernel(const float* __restrict__ qbar,
                                                     const float* __restrict__ kbar,
                                                     float* __restrict__ S, int Nb, int d) {
  __shared__ float Qs[64][33];
  __shared__ float Ks[64][33];
  const int tx = threadIdx.x, ty = threadIdx.y, tid = ty * 16 + tx;
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64, bh = blockIdx.z;
  const float* qb = qbar + size_t(bh) * Nb * d;
  const float* kb = kbar + size_t(bh) * Nb * d;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
  for (int k0 = 0; k0 < d; k0 += 32) {
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int r = it * 8 + tid / 32, c = tid % 32;
      Qs[r][c] = (i0 + r < Nb) ? qb[size_t(i0 + r) * d + k0 + c] : 0.0f;
      Ks[r][c] = (j0 + r < Nb) ? kb[size_t(j0 + r) * d + k0 + c] : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      float qv[4], kv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) qv[a] = Qs[ty + 16 * a][kk];
#pragma unroll
      for (int b = 0; b < 4; ++b) kv[b] = Ks[tx + 16 * b][kk];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = __fadd_rn(acc[a][b], __fmul_rn(qv[a], kv[b]));
    }
    __syncthreads();
  }
  float* Sb = S + size_t(bh) * Nb * Nb;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty + 16 * a;
    if (i >= Nb) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = j0 + tx + 16 * b;
      if (j < Nb) Sb[size_t(i) * Nb + j] = acc[a][b];
    }
  }
}

cudaError_t launch_scores(const Layout& L, const float* qbar, const float* kbar, float* scores,
                          cudaStream_t s) {
  dim3 grid((L.Nb + 63) / 64, (L.Nb + 63) / 64, L.BH);
  scores_kernel<<<grid, dim3(16, 16), 0, s>>>(qbar, kbar, scores, L.Nb, L.d);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// classification
// ---------------------------------------------------------------------------
constexpr int kClsThreads = 256;

// Monotone map float -> uint32 (larger float, larger key); -0 and +0 map alike.
__device__ __forceinline__ uint32_t order_key(float s) {
  const uint32_t u = __float_as_uint(__fadd_rn(s, 0.0f));
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum of `v` over the CTA's threads in thread order.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < wid; ++w) base += warp_tot[w];
  __syncthreads();
  return base + incl - v;
}

// k-th largest key (k >= 1) by 4 passes of an 8-bit radix select. Returns the
// key value T and `need`, the number of elements equal to T that belong to
// the top k (the others above T are all in it).
__device__ void radix_select_top(const uint32_t* keys, int lo, int hi, int k, int* hist, int* sel,
                                 uint32_t& T, int& need) {
  uint32_t prefix = 0, pmask = 0;
  int rem = k;
  const int tid = threadIdx.x, lane = tid & 31;
  for (int shift = 24; shift >= 0; shift -= 8) {
    hist[tid] = 0;  // kClsThreads == 256 bins
    __syncthreads();
    for (int j = lo; j < hi; ++j) {
      const uint32_t key = keys[j];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid < 32) {
      int c[8], sum = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = hist[255 - 8 * lane - e];
        sum += c[e];
      }
      int incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= rem);
      if (lane == __ffs(hit) - 1) {
        int cum = incl - sum;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (cum + c[e] >= rem) {
            sel[0] = 255 - 8 * lane - e;
            sel[1] = rem - cum;
            break;
          }
          cum += c[e];
        }
      }
    }
    __syncthreads();
    prefix |= uint32_t(sel[0]) << shift;
    pmask |= 0xFFu << shift;
    rem = sel[1];
    __syncthreads();
  }
  T = prefix;
  need = rem;
}

// One CTA per (bh, query block i). Top k_crit by (score desc, index asc) are
// critical; elements outside the top (Nb - k_neg) are negligible.
__global__ void __launch_bounds__(kClsThreads) classify_kernel(const float* __restrict__ S,
                                                               int8_t* __restrict__ Mc,
                                                               int32_t* __restrict__ crit,
                                                               int32_t* __restrict__ neg, int Nb,
                                                               int kc, int kn) {
  __shared__ uint32_t keys[SLA_MAX_BLOCKS];
  __shared__ int hist[256];
  __shared__ int sel[2];
  __shared__ int warp_tot[kClsThreads / 32];
  const size_t row = size_t(blockIdx.y) * Nb + blockIdx.x;
  const float* srow = S + row * Nb;
  const int E = (Nb + kClsThreads - 1) / kClsThreads;
  const int lo = min(Nb, int(threadIdx.x) * E), hi = min(Nb, lo + E);
  for (int j = threadIdx.x; j < Nb; j += kClsThreads) keys[j] = order_key(srow[j]);
  __syncthreads();

  // top k_crit
  uint32_t Tc;
  int needc;
  radix_select_top(keys, lo, hi, kc, hist, sel, Tc, needc);
  int eq = 0;
  for (int j = lo; j < hi; ++j) eq += keys[j] == Tc;
  int eqrank = block_exclusive_scan(eq, warp_tot);
  // top (Nb - k_neg): everything else is negligible
  uint32_t Tn = 0;
  int needn = 0, eqrank_n = 0;
  if (kn > 0) {
    radix_select_top(keys, lo, hi, Nb - kn, hist, sel, Tn, needn);
    int eqn = 0;
    for (int j = lo; j < hi; ++j) eqn += keys[j] == Tn;
    eqrank_n = block_exclusive_scan(eqn, warp_tot);
  }
  // labels
  int8_t* mrow = Mc + row * Nb;
  int ncrit = 0, nneg = 0;
  for (int j = lo; j < hi; ++j) {
    const uint32_t key = keys[j];
    bool c = key > Tc || (key == Tc && eqrank < needc);
    eqrank += key == Tc;
    bool n = false;
    if (kn > 0) {
      const bool top = key > Tn || (key == Tn && eqrank_n < needn);
      eqrank_n += key == Tn;
      n = !top;
    }
    mrow[j] = c ? int8_t(1) : (n ? int8_t(-1) : int8_t(0));
    ncrit += c;
    nneg += n;
  }
  // ascending index lists
  int pc = block_exclusive_scan(ncrit, warp_tot);
  int pn = block_exclusive_scan(nneg, warp_tot);
  int32_t* crow = crit + row * kc;
  int32_t* nrow = neg + row * (kn > 0 ? kn : 1);
  for (int j = lo; j < hi; ++j) {
    const int8_t m = mrow[j];
    if (m == 1) {
      if (pc < kc) crow[pc] = j;  // exactly k_crit labels exist; the bound is defensive
      ++pc;
    } else if (m == -1) {
      if (pn < kn) nrow[pn] = j;
      ++pn;
    }
  }
}

cudaError_t launch_classify(const Layout& L, const float* scores, int8_t* mc, int32_t* crit,
                            int32_t* neg, cudaStream_t s) {
  dim3 grid(L.Nb, L.BH);
  classify_kernel<<<grid, kClsThreads, 0, s>>>(scores, mc, crit, neg, L.Nb, L.kc, L.kn);
  return cudaGetLastError();
}

}  // namespace sla
