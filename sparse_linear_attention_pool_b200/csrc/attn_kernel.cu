// Hybrid compute and fusion (step 4 of the forward), one CTA per (64-row
// query block i, head):
//   sparse branch  O^s_i = softmax over the keys of the critical blocks of row i
//                  (online softmax, scale 1/sqrt(d)), SLA structured summary
//                  (aipaper.cc) section 4 step 3; walkthrough (intelliparadigm.com)
//                  section 2.2 (online softmax, bq = bkv = 64);
//   linear branch  O^l_i = phi(Q_i) H_i / phi(Q_i) Z_i over the marginal blocks,
//                  summary section 4 formula 3, with
//                  H_i = H_tot - sum_{j in E_i} phi(K_j)^T V_j and
//                  Z_i = Z_tot - sum_{j in E_i} rowsum(phi(K_j)^T), E_i the
//                  critical and negligible blocks of row i; the excluded terms
//                  enter as phi(Q_i) phi(K_j)^T V_j, computed from the K/V tiles;
//   combine        SLA: O = O^s + O^l W (summary formula 4);
//                  SLA2: O = alpha_h O^s + (1 - alpha_h) O^l (SLA2 article,
//                  mcffsbgs.com, mixing-formula paragraph).
// Dense mode (the baseline): every key block critical, no linear branch.
//
// Tensor-core products use mma.sync m16n8k16 (bf16 inputs, fp32 accumulate);
// 4 warps, each owning 16 query rows; K/V tiles double-buffered with cp.async.
#include "sla_internal.cuh"

namespace sla {

template <int D>
struct AttnSmem {
  static constexpr int kTile = 64 * D;  // bf16 elements of a 64-row tile
  static constexpr size_t q = 0;
  static constexpr size_t pq = q + kTile * 2;
  static constexpr size_t k = pq + kTile * 2;         // 2 buffers (also H_tot later)
  static constexpr size_t v = k + 2 * kTile * 2;      // 2 buffers (also W later)
  static constexpr size_t stash = v + 2 * kTile * 2;  // O^s, fp32, fragment order
  static constexpr size_t den = stash + kTile * 4;
  static constexpr size_t bytes = den + 64 * 4;
};

// rows x D bf16 tile from global (row stride D) into swizzled shared memory;
// rows >= valid are zero-filled.
template <int D>
__device__ __forceinline__ void load_tile(__nv_bfloat16* sm, const __nv_bfloat16* g, int rows,
                                          int valid) {
  constexpr int CPR = D / 8;
  for (int id = threadIdx.x; id < rows * CPR; id += blockDim.x) {
    const int r = id / CPR, ch = id % CPR;
    const bool v = r < valid;
    cp_async16(smem_u32(sm + r * D + ((ch ^ (r & 7)) << 3)),
               v ? (const void*)(g + size_t(r) * D + ch * 8) : (const void*)g, v);
  }
}

// S[16 x 64] (this warp's rows) = A[16 x D] * B[64 x D]^T from swizzled tiles.
template <int D>
__device__ __forceinline__ void warp_qk(float (&s)[8][4], const __nv_bfloat16* A,
                                        const __nv_bfloat16* B, int warp, int lane) {
#pragma unroll
  for (int t = 0; t < 8; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[t][e] = 0.0f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4];
    ldsm_x4(smem_u32(A + swz(16 * warp + (lane & 7) + (((lane >> 3) & 1) << 3),
                             16 * kk + ((lane >> 4) << 3), D)),
            a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(smem_u32(B + swz(16 * p + (lane & 7) + ((lane >> 4) << 3),
                               16 * kk + (((lane >> 3) & 1) << 3), D)),
              b0, b1, b2, b3);
      mma16816(s[2 * p], a, b0, b1);
      mma16816(s[2 * p + 1], a, b2, b3);
    }
  }
}

// acc[16 x D] += P[16 x 64] (bf16, from registers) * Vt[64 x D] (swizzled tile).
template <int D>
__device__ __forceinline__ void warp_pv(float (&acc)[D / 8][4], const float (&p)[8][4],
                                        const __nv_bfloat16* Vt, int lane) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t a[4];
    a[0] = pack_bf16(p[2 * kk][0], p[2 * kk][1]);
    a[1] = pack_bf16(p[2 * kk][2], p[2 * kk][3]);
    a[2] = pack_bf16(p[2 * kk + 1][0], p[2 * kk + 1][1]);
    a[3] = pack_bf16(p[2 * kk + 1][2], p[2 * kk + 1][3]);
#pragma unroll
    for (int q = 0; q < D / 16; ++q) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(Vt + swz(16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3),
                                  16 * q + ((lane >> 4) << 3), D)),
                b0, b1, b2, b3);
      mma16816(acc[2 * q], a, b0, b1);
      mma16816(acc[2 * q + 1], a, b2, b3);
    }
  }
}

// acc[16 x D] += A[16 x D] (swizzled tile, this warp's rows) * M[D x D] (swizzled, row = k).
template <int D>
__device__ __forceinline__ void warp_a_mat(float (&acc)[D / 8][4], const __nv_bfloat16* A,
                                           const __nv_bfloat16* M, int warp, int lane) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4];
    ldsm_x4(smem_u32(A + swz(16 * warp + (lane & 7) + (((lane >> 3) & 1) << 3),
                             16 * kk + ((lane >> 4) << 3), D)),
            a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int q = 0; q < D / 16; ++q) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(M + swz(16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3),
                                 16 * q + ((lane >> 4) << 3), D)),
                b0, b1, b2, b3);
      mma16816(acc[2 * q], a, b0, b1);
      mma16816(acc[2 * q + 1], a, b2, b3);
    }
  }
}

template <int D, int MODE>
__global__ void __launch_bounds__(128, 1) attn_kernel(const AttnArgs a) {
  using SM = AttnSmem<D>;
  constexpr int kTile = SM::kTile;
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(smem + SM::q);
  __nv_bfloat16* PQs = reinterpret_cast<__nv_bfloat16*>(smem + SM::pq);
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smem + SM::k);
  __nv_bfloat16* Vs = reinterpret_cast<__nv_bfloat16*>(smem + SM::v);
  float* stash = reinterpret_cast<float*>(smem + SM::stash);
  float* den = reinterpret_cast<float*>(smem + SM::den);

  const int i = blockIdx.x, bh = blockIdx.y, h = bh % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N, Nb = a.Nb;
  const int Npad = Nb * kBlock;
  const size_t hoff = size_t(bh) * Npad * D;
  const int row0 = i * kBlock;
  const int nq = min(kBlock, N - row0);
  const int32_t* crow = a.crit + (size_t(bh) * Nb + i) * a.kc;
  const int32_t* nrow = a.neg + (size_t(bh) * Nb + i) * (a.kn > 0 ? a.kn : 1);
  const int nA = MODE == kModeDense ? Nb : a.kc;
  // Block indices from the lists are clamped into [0, Nb): a bad list entry is
  // reported through the status word instead of becoming an out-of-bounds load.
  auto checked = [&](int j) {
    if (j < 0 || j >= Nb) {
      if (a.status) *a.status = kDevBadIndex;
      j = j < 0 ? 0 : Nb - 1;
    }
    return j;
  };
  auto blockA = [&](int idx) { return MODE == kModeDense ? idx : checked(crow[idx]); };

  load_tile<D>(Qs, a.Q + hoff + size_t(row0) * D, 64, nq);
  cp_async_commit();
  {
    const int j = blockA(0);
    load_tile<D>(Ks, a.K + hoff + size_t(j) * kBlock * D, 64, min(kBlock, N - j * kBlock));
    load_tile<D>(Vs, a.V + hoff + size_t(j) * kBlock * D, 64, min(kBlock, N - j * kBlock));
  }
  cp_async_commit();
  cp_async_wait<1>();
  __syncthreads();

  if (MODE != kModeDense) {
    // phi(Q_i) rows -> PQs (bf16); den[r] = phi(q_r) . Z_tot with the rounded phi values
    constexpr int PL = D / 32;
    const float* zt = a.ztot + size_t(bh) * D;
    for (int r = warp; r < 64; r += 4) {
      const int col = lane * PL;
      float x[PL];
#pragma unroll
      for (int e = 0; e < PL; ++e) x[e] = bf2f(Qs[swz(r, col + e, D)]);
      float dsum = 0.0f;
      if (r < nq) {
        float m = -INFINITY;
#pragma unroll
        for (int e = 0; e < PL; ++e) m = fmaxf(m, x[e]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float s = 0.0f;
#pragma unroll
        for (int e = 0; e < PL; ++e) {
          x[e] = expf(x[e] - m);
          s += x[e];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        const float inv = 1.0f / s;
#pragma unroll
        for (int e = 0; e < PL; ++e) x[e] *= inv;
      } else {
#pragma unroll
        for (int e = 0; e < PL; ++e) x[e] = 0.0f;
      }
#pragma unroll
      for (int e = 0; e < PL; e += 2) {
        const uint32_t pk = pack_bf16(x[e], x[e + 1]);
        *reinterpret_cast<uint32_t*>(PQs + swz(r, col + e, D)) = pk;
        dsum += bf16_lo(pk) * zt[col + e] + bf16_hi(pk) * zt[col + e + 1];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
      if (lane == 0) den[r] = dsum;
    }
  }

  // ---------------- sparse branch over the critical blocks ----------------
  float o[D / 8][4];
#pragma unroll
  for (int t = 0; t < D / 8; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[t][e] = 0.0f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.0f, 0.0f};
  const float sl2 = a.scale_log2;
  for (int it = 0; it < nA; ++it) {
    const int buf = it & 1;
    if (it + 1 < nA) {
      const int jn = blockA(it + 1);
      const int nvn = min(kBlock, N - jn * kBlock);
      load_tile<D>(Ks + (buf ^ 1) * kTile, a.K + hoff + size_t(jn) * kBlock * D, 64, nvn);
      load_tile<D>(Vs + (buf ^ 1) * kTile, a.V + hoff + size_t(jn) * kBlock * D, 64, nvn);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    float s[8][4];
    warp_qk<D>(s, Qs, Ks + buf * kTile, warp, lane);
    const int j = blockA(it);
    if (j * kBlock + kBlock > N) {  // partial last block: mask pad keys
#pragma unroll
      for (int t = 0; t < 8; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (j * kBlock + 8 * t + 2 * (lane & 3) + (e & 1) >= N) s[t][e] = -INFINITY;
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mx = -INFINITY;
#pragma unroll
      for (int t = 0; t < 8; ++t) mx = fmaxf(mx, fmaxf(s[t][2 * r], s[t][2 * r + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(mrow[r], mx * sl2);
      const float corr = exp2f(mrow[r] - mnew);
      mrow[r] = mnew;
      float rs = 0.0f;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        s[t][2 * r] = exp2f(s[t][2 * r] * sl2 - mnew);
        s[t][2 * r + 1] = exp2f(s[t][2 * r + 1] * sl2 - mnew);
        rs += s[t][2 * r] + s[t][2 * r + 1];
      }
      lrow[r] = lrow[r] * corr + rs;
#pragma unroll
      for (int t = 0; t < D / 8; ++t) {
        o[t][2 * r] *= corr;
        o[t][2 * r + 1] *= corr;
      }
    }
    warp_pv<D>(o, s, Vs + buf * kTile, lane);
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
    const float inv = 1.0f / lrow[r];
#pragma unroll
    for (int t = 0; t < D / 8; ++t) {
      o[t][2 * r] *= inv;
      o[t][2 * r + 1] *= inv;
    }
  }
  const int r_lo = 16 * warp + (lane >> 2);  // this thread's two rows: r_lo, r_lo + 8
  __nv_bfloat16* Og = a.O + hoff + size_t(row0) * D;

  if (MODE == kModeDense) {
#pragma unroll
    for (int t = 0; t < D / 8; ++t) {
      const int c = 8 * t + 2 * (lane & 3);
      if (r_lo < nq) *reinterpret_cast<uint32_t*>(Og + size_t(r_lo) * D + c) = pack_bf16(o[t][0], o[t][1]);
      if (r_lo + 8 < nq)
        *reinterpret_cast<uint32_t*>(Og + size_t(r_lo + 8) * D + c) = pack_bf16(o[t][2], o[t][3]);
    }
    return;
  }

  // keep O^s in shared memory while the linear branch runs
#pragma unroll
  for (int t = 0; t < D / 8; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) stash[((warp * (D / 8) + t) * 4 + e) * 32 + lane] = o[t][e];

  // ---------------- linear branch ----------------
  const bool has_marg = a.kc + a.kn < Nb;
  float c[D / 8][4];  // correction sum_{j in E} phi(Q) phi(K_j)^T V_j, then the numerator
#pragma unroll
  for (int t = 0; t < D / 8; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) c[t][e] = 0.0f;
  float dc[2] = {0.0f, 0.0f};
  if (has_marg) {
    const int nE = a.kc + a.kn;
    auto blockE = [&](int idx) { return checked(idx < a.kc ? crow[idx] : nrow[idx - a.kc]); };
    {
      const int j = blockE(0);
      load_tile<D>(Ks, a.phik + hoff + size_t(j) * kBlock * D, 64, kBlock);
      load_tile<D>(Vs, a.V + hoff + size_t(j) * kBlock * D, 64, min(kBlock, N - j * kBlock));
    }
    cp_async_commit();
    for (int it = 0; it < nE; ++it) {
      const int buf = it & 1;
      if (it + 1 < nE) {
        const int jn = blockE(it + 1);
        load_tile<D>(Ks + (buf ^ 1) * kTile, a.phik + hoff + size_t(jn) * kBlock * D, 64, kBlock);
        load_tile<D>(Vs + (buf ^ 1) * kTile, a.V + hoff + size_t(jn) * kBlock * D, 64,
                     min(kBlock, N - jn * kBlock));
      }
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      float f[8][4];
      warp_qk<D>(f, PQs, Ks + buf * kTile, warp, lane);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        dc[0] += f[t][0] + f[t][1];
        dc[1] += f[t][2] + f[t][3];
      }
      warp_pv<D>(c, f, Vs + buf * kTile, lane);
      __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      dc[r] += __shfl_xor_sync(0xffffffffu, dc[r], 1);
      dc[r] += __shfl_xor_sync(0xffffffffu, dc[r], 2);
    }
    // numerator = phi(Q) H_tot - correction
    load_tile<D>(Ks, a.htot16 + size_t(bh) * D * D, D, D);
  }
  const bool use_w = MODE == kModeSLA && a.w_proj != nullptr;
  if (use_w) load_tile<D>(Vs, a.w_proj, D, D);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  if (has_marg) {
#pragma unroll
    for (int t = 0; t < D / 8; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) c[t][e] = -c[t][e];
    warp_a_mat<D>(c, PQs, Ks, warp, lane);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float inv = 1.0f / (den[r_lo + 8 * r] - dc[r]);
#pragma unroll
      for (int t = 0; t < D / 8; ++t) {
        c[t][2 * r] *= inv;
        c[t][2 * r + 1] *= inv;
      }
    }
  }
  // c now holds O^l (zero when the marginal set is empty)
  float alpha = 0.0f;
  if (MODE == kModeSLA2) alpha = a.alpha[h];
  if (use_w) {
    uint32_t ol[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      ol[kk][0] = pack_bf16(c[2 * kk][0], c[2 * kk][1]);
      ol[kk][1] = pack_bf16(c[2 * kk][2], c[2 * kk][3]);
      ol[kk][2] = pack_bf16(c[2 * kk + 1][0], c[2 * kk + 1][1]);
      ol[kk][3] = pack_bf16(c[2 * kk + 1][2], c[2 * kk + 1][3]);
    }
#pragma unroll
    for (int t = 0; t < D / 8; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) c[t][e] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int q = 0; q < D / 16; ++q) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(Vs + swz(16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3),
                                    16 * q + ((lane >> 4) << 3), D)),
                  b0, b1, b2, b3);
        mma16816(c[2 * q], ol[kk], b0, b1);
        mma16816(c[2 * q + 1], ol[kk], b2, b3);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < D / 8; ++t) {
    float out[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float os = stash[((warp * (D / 8) + t) * 4 + e) * 32 + lane];
      out[e] = MODE == kModeSLA2 ? alpha * os + (1.0f - alpha) * c[t][e] : os + c[t][e];
    }
    const int col = 8 * t + 2 * (lane & 3);
    if (r_lo < nq) *reinterpret_cast<uint32_t*>(Og + size_t(r_lo) * D + col) = pack_bf16(out[0], out[1]);
    if (r_lo + 8 < nq)
      *reinterpret_cast<uint32_t*>(Og + size_t(r_lo + 8) * D + col) = pack_bf16(out[2], out[3]);
  }
}

template <int D, int MODE>
static cudaError_t launch_t(const AttnArgs& a, int BH, cudaStream_t s) {
  const size_t bytes = AttnSmem<D>::bytes;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
  if (e != cudaSuccess) return e;
  attn_kernel<D, MODE><<<dim3(a.Nb, BH), 128, bytes, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_attention(const AttnArgs& a, int BH, int d, int mode, cudaStream_t s) {
  if (d == 128) {
    if (mode == kModeSLA) return launch_t<128, kModeSLA>(a, BH, s);
    if (mode == kModeSLA2) return launch_t<128, kModeSLA2>(a, BH, s);
    return launch_t<128, kModeDense>(a, BH, s);
  }
  if (mode == kModeSLA) return launch_t<64, kModeSLA>(a, BH, s);
  if (mode == kModeSLA2) return launch_t<64, kModeSLA2>(a, BH, s);
  return launch_t<64, kModeDense>(a, BH, s);
}

}  // namespace sla
