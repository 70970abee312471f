// Linear-attention precompute (step 3 of the forward): phi(K) with
// phi = softmax over the head dimension (or, selected by the caller, elu + 1
// elementwise: SLA structured summary, section 4), the per-block column sums
// z_j = rowsum(phi(K_j)^T), and the per-head totals
// H_tot = sum_j phi(K_j)^T V_j, Z_tot = sum_j z_j.
//
// Source: SLA walkthrough (intelliparadigm.com), section 1.2 ("precompute
// h_j = phi(K_j)^T V_j and z_j = rowsum(phi(K_j)^T)") and section 2.2
// (the H / Z accumulation pseudo-code); SLA structured summary (aipaper.cc),
// section 4, formula 3; phi = softmax: walkthrough section 3.2.
//
// The per-query-block sums over marginal blocks are formed later as
// H_i = H_tot - sum_{j excluded from row i} h_j (likewise Z_i), with the
// excluded (critical and negligible) blocks' terms recomputed from the tiles
// the attention kernel loads, so H_tot / Z_tot and z_j are all that is stored
// here besides phi(K). Reductions run in a fixed order (no atomics): results
// are deterministic.
#include "sla_internal.cuh"

namespace sla {

// CTA of 256 threads (8 warps) per (1024-token chunk, head). The K and V
// tiles of the next 64-token block stream in (cp.async, double-buffered)
// while the current one is processed: phi(K) rows -> shared memory and global
// (bf16), z_j -> global, H_chunk += phi(K_j)^T V_j on tensor cores
// (mma.sync m16n8k16, fp32 accumulation).
template <int D>
__global__ void __launch_bounds__(256) phik_hz_kernel(const __nv_bfloat16* __restrict__ K,
                                                      const __nv_bfloat16* __restrict__ V,
                                                      __nv_bfloat16* __restrict__ phik,
                                                      float* __restrict__ zblk,
                                                      float* __restrict__ hpart, float* __restrict__ zpart,
                                                      uint8_t* __restrict__ vcode,
                                                      float* __restrict__ vscale, int phi_elu1, int N,
                                                      int Npad, int Nb, int nchunk) {
  __shared__ float vred[8];
  constexpr int CPR = D / 8;    // 16-byte chunks per row
  constexpr int WPM = 128 / D;  // warps per 16-row m tile (1 for D=128, 2 for D=64)
  constexpr int NCOL = D / WPM; // output columns per warp
  constexpr int NT = NCOL / 8;  // n tiles per warp
  constexpr int kT = 64 * D;    // elements of a 64-row tile
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smem_raw);  // [2][64 x D]
  __nv_bfloat16* Vs = Ks + 2 * kT;                                  // [2][64 x D]
  __nv_bfloat16* PK = Vs + 2 * kT;                                  // [64 x D]
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = warp / WPM, n0 = (warp % WPM) * NCOL;
  const size_t hoff = size_t(bh) * Npad * D;
  const int jb0 = chunk * (kHzChunk / kBlock);
  const int jb1 = min(Nb, jb0 + kHzChunk / kBlock);

  auto load_block = [&](int jb, int buf) {
    const int t0 = jb * kBlock;
    const int nv = min(kBlock, N - t0);
    for (int id = threadIdx.x; id < 64 * CPR; id += 256) {
      const int r = id / CPR, ch = id % CPR;
      const bool v = r < nv;  // rows past N are zero-filled, never read
      const size_t g = hoff + size_t(t0 + r) * D + ch * 8;
      const int s = r * D + ((ch ^ (r & 7)) << 3);
      cp_async16(smem_u32(Ks + buf * kT + s), v ? (const void*)(K + g) : (const void*)K, v);
      cp_async16(smem_u32(Vs + buf * kT + s), v ? (const void*)(V + g) : (const void*)V, v);
    }
  };

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[t][e] = 0.0f;
  float zsum[2] = {0.0f, 0.0f};

  load_block(jb0, 0);
  cp_async_commit();
  for (int jb = jb0; jb < jb1; ++jb) {
    const int buf = (jb - jb0) & 1;
    const int t0 = jb * kBlock;
    const int nv = min(kBlock, N - t0);
    if (jb + 1 < jb1) load_block(jb + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    // phi(K) rows: warp w handles rows w, w+8, ...; a lane holds D/32 columns
    const __nv_bfloat16* Kb = Ks + buf * kT;
    constexpr int PL = D / 32;
    const int col = lane * PL;
    for (int r = warp; r < 64; r += 8) {
      float x[PL];
      if (r < nv) {
        const __nv_bfloat16* src = Kb + swz(r, col, D);
        if constexpr (PL == 4) {
          const uint2 raw = *reinterpret_cast<const uint2*>(src);
          x[0] = bf16_lo(raw.x);
          x[1] = bf16_hi(raw.x);
          x[2] = bf16_lo(raw.y);
          x[3] = bf16_hi(raw.y);
        } else {
          const uint32_t raw = *reinterpret_cast<const uint32_t*>(src);
          x[0] = bf16_lo(raw);
          x[1] = bf16_hi(raw);
        }
        if (phi_elu1) {  // elu(x) + 1, elementwise
#pragma unroll
          for (int e = 0; e < PL; ++e) x[e] = x[e] > 0.0f ? x[e] + 1.0f : expf(x[e]);
        } else {  // softmax over the row (the warp's 32 lanes)
          float m = x[0];
#pragma unroll
          for (int e = 1; e < PL; ++e) m = fmaxf(m, x[e]);
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
        }
      } else {
#pragma unroll
        for (int e = 0; e < PL; ++e) x[e] = 0.0f;
      }
      uint32_t pk[PL / 2];
#pragma unroll
      for (int e = 0; e < PL / 2; ++e) pk[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
      __nv_bfloat16* sdst = PK + swz(r, col, D);
      __nv_bfloat16* gdst = phik + hoff + size_t(t0 + r) * D + col;
      if constexpr (PL == 4) {
        *reinterpret_cast<uint2*>(sdst) = make_uint2(pk[0], pk[1]);
        *reinterpret_cast<uint2*>(gdst) = make_uint2(pk[0], pk[1]);
      } else {
        *reinterpret_cast<uint32_t*>(sdst) = pk[0];
        *reinterpret_cast<uint32_t*>(gdst) = pk[0];
      }
    }
    if (vcode != nullptr) {
      // FP8 e4m3 form of V for the quantised sparse branch: scale absmax / 448
      // over the block (s = 1 when absmax = 0), code = e4m3(v / s), round to
      // nearest even, saturating; rows >= N are zero in the tile.
      const __nv_bfloat16* Vt = Vs + buf * kT;
      constexpr int kChunks = 64 * CPR / 256;  // 16-byte chunks per thread
      float amax = 0.0f;
#pragma unroll
      for (int k = 0; k < kChunks; ++k) {
        const int ch = threadIdx.x + 256 * k, r = ch / CPR, cc = ch % CPR;
        const uint4 raw = *reinterpret_cast<const uint4*>(Vt + r * D + ((cc ^ (r & 7)) << 3));
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[e])), fabsf(bf16_hi(w[e]))));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      if (lane == 0) vred[warp] = amax;
      __syncthreads();
      amax = vred[0];
#pragma unroll
      for (int w8 = 1; w8 < 8; ++w8) amax = fmaxf(amax, vred[w8]);
      const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
      if (threadIdx.x == 0) vscale[size_t(bh) * Nb + jb] = s;
      uint8_t* vb = vcode + hoff + size_t(t0) * D;
#pragma unroll
      for (int k = 0; k < kChunks; ++k) {
        const int ch = threadIdx.x + 256 * k, r = ch / CPR, cc = ch % CPR;
        const uint4 raw = *reinterpret_cast<const uint4*>(Vt + r * D + ((cc ^ (r & 7)) << 3));
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t p[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          p[e >> 1] |= pack_e4m3x2(__fdiv_rn(bf16_lo(w[e]), s), __fdiv_rn(bf16_hi(w[e]), s)) << (16 * (e & 1));
        *reinterpret_cast<uint2*>(vb + size_t(r) * D + cc * 8) = make_uint2(p[0], p[1]);
      }
    }
    __syncthreads();
    // H_chunk += phi(K_j)^T V_j : A = phi(K)^T (m = dim, k = token), B = V.
    // z_j = phi(K_j)^T 1 rides along as one more n-tile with B = all ones.
    const __nv_bfloat16* Vb = Vs + buf * kT;
    float zacc[4] = {0.f, 0.f, 0.f, 0.f};
    constexpr uint32_t kOnes = 0x3F803F80u;  // bf16x2 (1.0, 1.0)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      {
        const int tr = 16 * kk + (lane & 7) + ((lane >> 4) << 3);
        const int tc = 16 * mt + (((lane >> 3) & 1) << 3);
        ldsm_x4_t(smem_u32(PK + swz(tr, tc, D)), a[0], a[1], a[2], a[3]);
      }
      if (n0 == 0) mma16816(zacc, a, kOnes, kOnes);
#pragma unroll
      for (int q = 0; q < NT / 2; ++q) {
        uint32_t b0, b1, b2, b3;
        const int tr = 16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int tc = n0 + 16 * q + ((lane >> 4) << 3);
        ldsm_x4_t(smem_u32(Vb + swz(tr, tc, D)), b0, b1, b2, b3);
        mma16816(acc[2 * q], a, b0, b1);
        mma16816(acc[2 * q + 1], a, b2, b3);
      }
    }
    if (n0 == 0 && (lane & 3) == 0) {  // every column of the ones-tile holds the row sum
      float* zdst = zblk + (size_t(bh) * Nb + jb) * D + 16 * mt + (lane >> 2);
      zdst[0] = zacc[0];
      zdst[8] = zacc[2];
      zsum[0] += zacc[0];  // chunk partial of Z_tot, blocks in ascending order
      zsum[1] += zacc[2];
    }
    __syncthreads();
  }
  if (n0 == 0 && (lane & 3) == 0) {
    float* zdst = zpart + (size_t(bh) * nchunk + chunk) * D + 16 * mt + (lane >> 2);
    zdst[0] = zsum[0];
    zdst[8] = zsum[1];
  }
  // partial H of this chunk: rows (dims) 16 mt + lane/4 (+8), columns n0 + 8t + 2(lane%4)
  float* hp = hpart + (size_t(bh) * nchunk + chunk) * D * D;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int r = 16 * mt + (lane >> 2);
    const int c = n0 + 8 * t + 2 * (lane & 3);
    *reinterpret_cast<float2*>(hp + size_t(r) * D + c) = make_float2(acc[t][0], acc[t][1]);
    *reinterpret_cast<float2*>(hp + size_t(r + 8) * D + c) = make_float2(acc[t][2], acc[t][3]);
  }
}

template <int D>
static cudaError_t launch_hz_t(const Layout& L, const __nv_bfloat16* K, const __nv_bfloat16* V,
                               __nv_bfloat16* phik, float* zblk, float* hpart, float* zpart,
                               uint8_t* vcode, float* vscale, int phi_elu1, cudaStream_t s) {
  const int bytes = 5 * 64 * D * 2;
  cudaError_t e =
      cudaFuncSetAttribute(phik_hz_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  phik_hz_kernel<D><<<dim3(L.nchunk, L.BH), 256, bytes, s>>>(K, V, phik, zblk, hpart, zpart, vcode, vscale,
                                                            phi_elu1, L.N, L.Npad, L.Nb, L.nchunk);
  return cudaGetLastError();
}

cudaError_t launch_phik_hz(const Layout& L, const __nv_bfloat16* K, const __nv_bfloat16* V,
                           __nv_bfloat16* phik, float* zblk, float* hpart, float* zpart,
                           uint8_t* vcode, float* vscale, int phi_elu1, cudaStream_t s) {
  return L.d == 128 ? launch_hz_t<128>(L, K, V, phik, zblk, hpart, zpart, vcode, vscale, phi_elu1, s)
                    : launch_hz_t<64>(L, K, V, phik, zblk, hpart, zpart, vcode, vscale, phi_elu1, s);
}

// Fixed-order sum of n strided values: 8 interleaved partial sums (element i
// goes to partial i % 8), combined pairwise. Independent loads keep the
// memory pipe busy; the order is the same on every call.
__device__ __forceinline__ float strided_sum(const float* __restrict__ src, int n, size_t stride) {
  float p[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int i = 0;
  for (; i + 8 <= n; i += 8) {
#pragma unroll
    for (int k = 0; k < 8; ++k) p[k] += src[size_t(i + k) * stride];
  }
  for (int k = 0; i < n; ++i, ++k) p[k] += src[size_t(i) * stride];
  return ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
}

// H_tot and Z_tot = sums of the per-chunk partials (fixed order, see
// strided_sum). Blocks x < d*d/256 reduce H; the last block reduces Z.
__global__ void __launch_bounds__(256) hz_reduce_kernel(const float* __restrict__ zpart,
                                                        const float* __restrict__ hpart,
                                                        float* __restrict__ htot32,
                                                        __nv_bfloat16* __restrict__ htot16,
                                                        float* __restrict__ ztot, int nchunk, int d) {
  const int bh = blockIdx.y;
  const size_t dd = size_t(d) * d;
  const int nh = int((dd + 255) / 256);
  if (int(blockIdx.x) < nh) {
    const int e = blockIdx.x * 256 + threadIdx.x;
    if (e < int(dd)) {
      const float v = strided_sum(hpart + size_t(bh) * nchunk * dd + e, nchunk, dd);
      htot32[size_t(bh) * dd + e] = v;
      htot16[size_t(bh) * dd + e] = __float2bfloat16_rn(v);
    }
  } else if (threadIdx.x < d) {
    ztot[size_t(bh) * d + threadIdx.x] =
        strided_sum(zpart + size_t(bh) * nchunk * d + threadIdx.x, nchunk, size_t(d));
  }
}

cudaError_t launch_hz_reduce(const Layout& L, const float* zpart, const float* hpart, float* htot32,
                             __nv_bfloat16* htot16, float* ztot, cudaStream_t s) {
  dim3 grid((L.d * L.d + 255) / 256 + 1, L.BH);
  hz_reduce_kernel<<<grid, 256, 0, s>>>(zpart, hpart, htot32, htot16, ztot, L.nchunk, L.d);
  return cudaGetLastError();
}

// Z_i = Z_tot - sum over the excluded blocks of query block i (its critical
// blocks, then its negligible ones, in list order) of z_j: the denominator
// vector of the linear branch ([SLA-sum] formula 3, the sum over the marginal
// blocks formed as a complement). One warp per query block, d / 32 columns per
// lane. A list entry outside [0, Nb) is clamped and flagged in the status word.
__global__ void __launch_bounds__(256) zi_kernel(const int32_t* __restrict__ crit,
                                                 const int32_t* __restrict__ neg,
                                                 const float* __restrict__ zblk,
                                                 const float* __restrict__ ztot, float* __restrict__ zi,
                                                 int* status, int Nb, int kc, int kn, int d) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + warp, bh = blockIdx.y;
  if (i >= Nb) return;
  const int32_t* cl = crit + (size_t(bh) * Nb + i) * kc;
  const int32_t* nl = neg + (size_t(bh) * Nb + i) * (kn > 0 ? kn : 1);
  const float* zb = zblk + size_t(bh) * Nb * d;
  const int per = d / 32;
  float z[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) z[q] = q < per ? ztot[size_t(bh) * d + lane + 32 * q] : 0.0f;
  const int ne = kc + kn;
  // list entries 32 at a time (one per lane, broadcast), so the row loads of a
  // batch are independent of each other
  for (int u0 = 0; u0 < ne; u0 += 32) {
    const int u = u0 + lane;
    int my = 0;
    if (u < ne) {
      my = u < kc ? cl[u] : nl[u - kc];
      if (my < 0 || my >= Nb) {
        if (status != nullptr) atomicExch(status, kDevBadIndex);
        my = my < 0 ? 0 : Nb - 1;
      }
    }
    const int cnt = min(32, ne - u0);
#pragma unroll 8
    for (int k = 0; k < cnt; ++k) {
      const int j = __shfl_sync(0xffffffffu, my, k);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (q < per) z[q] -= zb[size_t(j) * d + lane + 32 * q];
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (q < per) zi[(size_t(bh) * Nb + i) * d + lane + 32 * q] = z[q];
}

cudaError_t launch_zi(const Layout& L, const int32_t* crit, const int32_t* neg, const float* zblk,
                      const float* ztot, float* zi, int* status, cudaStream_t s) {
  dim3 grid((L.Nb + 7) / 8, L.BH);
  zi_kernel<<<grid, 256, 0, s>>>(crit, neg, zblk, ztot, zi, status, L.Nb, L.kc, L.kn, L.d);
  return cudaGetLastError();
}

}  // namespace sla
