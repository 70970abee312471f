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
// With qcode != nullptr the same pass also writes the INT8 form of the block
// for the quantised sparse branch: scale s = absmax / 127 over the block's
// valid rows (s = 1 when absmax = 0), code = clamp(rint(x / s), -127, 127)
// with x / s one rounded float32 division (rows >= N get code 0).
template <int D, bool PHI>
__global__ void __launch_bounds__(128) pool_kernel(const __nv_bfloat16* __restrict__ Q,
                                                   const __nv_bfloat16* __restrict__ K,
                                                   const __nv_bfloat16* __restrict__ proj_q,
                                                   const __nv_bfloat16* __restrict__ proj_k,
                                                   float* __restrict__ qbar, float* __restrict__ kbar,
                                                   int8_t* __restrict__ qcode, int8_t* __restrict__ kcode,
                                                   float* __restrict__ qscale, float* __restrict__ kscale,
                                                   __nv_bfloat16* __restrict__ phiq, int phi_elu1, int N,
                                                   int Npad, int Nb) {
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
  int8_t* code = which == 0 ? qcode : kcode;
  float* cscale = which == 0 ? qscale : kscale;

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  float amax = 0.0f;
  const bool live = blk < Nb;
  // phi(Q) rows (softmax over the head dimension) for the linear branch; the
  // TPB threads of a row are contiguous lanes, reduced with shuffles inside
  // their group. Pad rows are not written (readers treat rows >= N as zero).
  const bool want_phi = PHI && which == 0;
  const unsigned gmask = (TPB == 32 ? 0xffffffffu : ((1u << TPB) - 1u)) << (threadIdx.x & 31 & ~(TPB - 1));
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
        amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[e])), fabsf(bf16_hi(w[e]))));
      }
      if (PHI && want_phi) {
        float x[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[2 * e] = bf16_lo(w[e]);
          x[2 * e + 1] = bf16_hi(w[e]);
        }
        float inv = 1.0f;
        if (phi_elu1) {  // elu(x) + 1, elementwise
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = x[e] > 0.0f ? x[e] + 1.0f : expf(x[e]);
        } else {  // softmax over the row (the group's TPB lanes)
          float m = x[0];
#pragma unroll
          for (int e = 1; e < 8; ++e) m = fmaxf(m, x[e]);
#pragma unroll
          for (int off = TPB / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(gmask, m, off));
          // exp(x - m) as 2^(x log2 e - m log2 e) on the MUFU ex2 unit
          const float ml = m * kLog2e;
          float sum = 0.0f;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            x[e] = ex2_approx(fmaf(x[e], kLog2e, -ml));
            sum += x[e];
          }
#pragma unroll
          for (int off = TPB / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(gmask, sum, off);
          inv = 1.0f / sum;
        }
        *reinterpret_cast<uint4*>(phiq + (size_t(bh) * Npad + size_t(blk) * kBlock + t) * D + c0) =
            make_uint4(pack_bf16(x[0] * inv, x[1] * inv), pack_bf16(x[2] * inv, x[3] * inv),
                       pack_bf16(x[4] * inv, x[5] * inv), pack_bf16(x[6] * inv, x[7] * inv));
      }
    }
  }
  if (code != nullptr) {
    // block absmax across the TPB threads of this block (contiguous lanes; all
    // threads take part, blocks past Nb contribute 0)
#pragma unroll
    for (int off = TPB / 2; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (live) {
      const int n = min(kBlock, N - blk * kBlock);
      const __nv_bfloat16* base = X + (size_t(bh) * Npad + size_t(blk) * kBlock) * D + c0;
      const float s = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 1.0f;
      if (threadIdx.x % TPB == 0) cscale[size_t(bh) * Nb + blk] = s;
      int8_t* cb = code + (size_t(bh) * Npad + size_t(blk) * kBlock) * D + c0;
      for (int t = 0; t < kBlock; ++t) {
        uint32_t lo = 0, hi = 0;
        if (t < n) {
          uint4 raw = *reinterpret_cast<const uint4*>(base + size_t(t) * D);
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
          int q8[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            q8[2 * e] = max(-127, min(127, __float2int_rn(__fdiv_rn(bf16_lo(w[e]), s))));
            q8[2 * e + 1] = max(-127, min(127, __float2int_rn(__fdiv_rn(bf16_hi(w[e]), s))));
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            lo |= uint32_t(q8[e] & 0xFF) << (8 * e);
            hi |= uint32_t(q8[4 + e] & 0xFF) << (8 * e);
          }
        }
        *reinterpret_cast<uint2*>(cb + size_t(t) * D) = make_uint2(lo, hi);
      }
    }
  }
  if (live) {
    const int n = min(kBlock, N - blk * kBlock);
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
                        float* kbar, int8_t* qcode, int8_t* kcode, float* qscale, float* kscale,
                        __nv_bfloat16* phiq, int phi_elu1, cudaStream_t s) {
  const int bpc = 128 / (L.d / 8);
  dim3 grid((L.Nb + bpc - 1) / bpc, L.BH, 2);
  // phi(Q) is a separate instantiation: the branch alone slows the plain pass
  if (L.d == 128) {
    if (phiq)
      pool_kernel<128, true><<<grid, 128, 0, s>>>(Q, K, proj_q, proj_k, qbar, kbar, qcode, kcode, qscale,
                                                  kscale, phiq, phi_elu1, L.N, L.Npad, L.Nb);
    else
      pool_kernel<128, false><<<grid, 128, 0, s>>>(Q, K, proj_q, proj_k, qbar, kbar, qcode, kcode, qscale,
                                                   kscale, nullptr, 0, L.N, L.Npad, L.Nb);
  } else {
    if (phiq)
      pool_kernel<64, true><<<grid, 128, 0, s>>>(Q, K, proj_q, proj_k, qbar, kbar, qcode, kcode, qscale,
                                                 kscale, phiq, phi_elu1, L.N, L.Npad, L.Nb);
    else
      pool_kernel<64, false><<<grid, 128, 0, s>>>(Q, K, proj_q, proj_k, qbar, kbar, qcode, kcode, qscale,
                                                  kscale, nullptr, 0, L.N, L.Npad, L.Nb);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// pooled scores
// ---------------------------------------------------------------------------
// CTA: 16 x 16 threads, a 64 x 128 tile of S; thread (tx, ty) owns rows
// ty + 16a (a < 4) and columns tx + 16b (b < 8). k runs ascending across
// 32-wide chunks; the next chunk's values are loaded into registers while the
// current one is multiplied, so the global loads overlap the arithmetic.
__global__ void __launch_bounds__(256) scores_kernel(const float* __restrict__ qbar,
                                                     const float* __restrict__ kbar,
                                                     float* __restrict__ S, int Nb, int d) {
  __shared__ float Qs[64][33];
  __shared__ float Ks[128][33];
  const int tx = threadIdx.x, ty = threadIdx.y, tid = ty * 16 + tx;
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 128, bh = blockIdx.z;
  const float* qb = qbar + size_t(bh) * Nb * d;
  const float* kb = kbar + size_t(bh) * Nb * d;
  float acc[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;
  // this thread's share of a chunk: rows it * 8 + tid / 32, column tid % 32
  float qn[8], kn[16];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int r = it * 8 + tid / 32, c = tid % 32;
      qn[it] = (i0 + r < Nb) ? qb[size_t(i0 + r) * d + k0 + c] : 0.0f;
    }
#pragma unroll
    for (int it = 0; it < 16; ++it) {
      const int r = it * 8 + tid / 32, c = tid % 32;
      kn[it] = (j0 + r < Nb) ? kb[size_t(j0 + r) * d + k0 + c] : 0.0f;
    }
  };
  fetch(0);
  for (int k0 = 0; k0 < d; k0 += 32) {
#pragma unroll
    for (int it = 0; it < 8; ++it) Qs[it * 8 + tid / 32][tid % 32] = qn[it];
#pragma unroll
    for (int it = 0; it < 16; ++it) Ks[it * 8 + tid / 32][tid % 32] = kn[it];
    __syncthreads();
    if (k0 + 32 < d) fetch(k0 + 32);
#pragma unroll 4
    for (int kk = 0; kk < 32; ++kk) {
      float qv[4], kv[8];
#pragma unroll
      for (int a = 0; a < 4; ++a) qv[a] = Qs[ty + 16 * a][kk];
#pragma unroll
      for (int b = 0; b < 8; ++b) kv[b] = Ks[tx + 16 * b][kk];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = __fadd_rn(acc[a][b], __fmul_rn(qv[a], kv[b]));
    }
    __syncthreads();
  }
  float* Sb = S + size_t(bh) * Nb * Nb;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty + 16 * a;
    if (i >= Nb) continue;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int j = j0 + tx + 16 * b;
      if (j < Nb) Sb[size_t(i) * Nb + j] = acc[a][b];
    }
  }
}

cudaError_t launch_scores(const Layout& L, const float* qbar, const float* kbar, float* scores,
                          cudaStream_t s) {
  dim3 grid((L.Nb + 127) / 128, (L.Nb + 63) / 64, L.BH);
  scores_kernel<<<grid, dim3(16, 16), 0, s>>>(qbar, kbar, scores, L.Nb, L.d);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// classification
// ---------------------------------------------------------------------------
// One warp per row (bh, query block i); 8 rows per CTA. The row's keys and a
// 256-bin histogram live in the warp's slice of shared memory; everything is
// warp-synchronous.
constexpr int kClsWarps = 8;

// Monotone map float -> uint32 (larger float, larger key); -0 and +0 map alike.
__device__ __forceinline__ uint32_t order_key(float s) {
  const uint32_t u = __float_as_uint(__fadd_rn(s, 0.0f));
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// k-th largest key (1 <= k <= n) by 4 passes of an 8-bit radix select. Returns
// the key value T and `need`, the number of elements equal to T that belong to
// the top k (every element above T is in it).
__device__ void warp_select_top(const uint32_t* keys, int n, int k, int* hist, uint32_t& T, int& need) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, pmask = 0;
  int rem = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j = lane; j < n; j += 32) {
      const uint32_t key = keys[j];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncwarp();
    // lane l scans bins 255-8l down to 248-8l (largest digits first)
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
    const int src = __ffs(hit) - 1;  // hit != 0: the total count n >= rem
    int sel = 0, nrem = 0;
    if (lane == src) {
      int cum = incl - sum;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (cum + c[e] >= rem) {
          sel = 255 - 8 * lane - e;
          nrem = rem - cum;
          break;
        }
        cum += c[e];
      }
    }
    sel = __shfl_sync(0xffffffffu, sel, src);
    rem = __shfl_sync(0xffffffffu, nrem, src);
    prefix |= uint32_t(sel) << shift;
    pmask |= 0xFFu << shift;
    __syncwarp();
  }
  T = prefix;
  need = rem;
}

// Top k_crit by (score desc, index asc) are critical; elements outside the
// top (Nb - k_neg) are negligible.
__global__ void __launch_bounds__(32 * kClsWarps) classify_kernel(const float* __restrict__ S,
                                                                  int8_t* __restrict__ Mc,
                                                                  int32_t* __restrict__ crit,
                                                                  int32_t* __restrict__ neg, int Nb,
                                                                  int kc, int kn, int rows) {
  extern __shared__ uint32_t cls_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_i = blockIdx.x * kClsWarps + warp;
  if (row_i >= rows) return;  // whole warp
  uint32_t* keys = cls_smem + size_t(warp) * (Nb + 256);
  int* hist = reinterpret_cast<int*>(keys + Nb);
  const size_t row = size_t(row_i);
  const float* srow = S + row * Nb;
  for (int j = lane; j < Nb; j += 32) keys[j] = order_key(srow[j]);
  __syncwarp();

  uint32_t Tc, Tn = 0;
  int needc, needn = 0;
  warp_select_top(keys, Nb, kc, hist, Tc, needc);
  if (kn > 0) warp_select_top(keys, Nb, Nb - kn, hist, Tn, needn);

  int8_t* mrow = Mc + row * Nb;
  int32_t* crow = crit + row * kc;
  int32_t* nrow = neg + row * (kn > 0 ? kn : 1);
  const unsigned lt = (1u << lane) - 1u;
  int eqc_seen = 0, eqn_seen = 0, ncrit = 0, nneg = 0;
  for (int base = 0; base < Nb; base += 32) {
    const int j = base + lane;
    const bool valid = j < Nb;
    const uint32_t key = valid ? keys[j] : 0u;
    const bool eqc = valid && key == Tc;
    const unsigned eqc_mask = __ballot_sync(0xffffffffu, eqc);
    const bool c = valid && (key > Tc || (eqc && eqc_seen + __popc(eqc_mask & lt) < needc));
    eqc_seen += __popc(eqc_mask);
    bool n = false;
    if (kn > 0) {
      const bool eqn = valid && key == Tn;
      const unsigned eqn_mask = __ballot_sync(0xffffffffu, eqn);
      const bool top = key > Tn || (eqn && eqn_seen + __popc(eqn_mask & lt) < needn);
      eqn_seen += __popc(eqn_mask);
      n = valid && !top;
    }
    if (valid) mrow[j] = c ? int8_t(1) : (n ? int8_t(-1) : int8_t(0));
    const unsigned cm = __ballot_sync(0xffffffffu, c);
    const unsigned nm = __ballot_sync(0xffffffffu, n);
    // exactly k_crit / k_neg labels exist; the bounds are defensive
    const int pc = ncrit + __popc(cm & lt), pn = nneg + __popc(nm & lt);
    if (c && pc < kc) crow[pc] = j;
    if (n && pn < kn) nrow[pn] = j;
    ncrit += __popc(cm);
    nneg += __popc(nm);
  }
}

cudaError_t launch_classify(const Layout& L, const float* scores, int8_t* mc, int32_t* crit,
                            int32_t* neg, cudaStream_t s) {
  const int rows = L.BH * L.Nb;
  const int bytes = kClsWarps * (L.Nb + 256) * 4;  // <= 8 * 4352 * 4 = 139264 for Nb <= 4096
  cudaError_t e = cudaFuncSetAttribute(classify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  classify_kernel<<<(rows + kClsWarps - 1) / kClsWarps, 32 * kClsWarps, bytes, s>>>(
      scores, mc, crit, neg, L.Nb, L.kc, L.kn, rows);
  return cudaGetLastError();
}

}  // namespace sla
