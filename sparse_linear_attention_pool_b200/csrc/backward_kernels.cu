// Backward pass of the SLA / SLA2 forward: gradients of <dO, O> with respect
// to Q, K, V (and SLA's W, SLA2's alpha) with the block mask held fixed.
//
// SLA walkthrough (intelliparadigm.com), section 2.3: the sparse path follows
// the FlashAttention backward on the Mc = 1 blocks; the linear path obtains
// the gradients of phi(Q), phi(K) and V by the chain rule, accumulated block
// by block. Written out (row r of query block i, key block j):
//   sparse:  P = exp(scale q.k - lse_r), D_r = dO^s_r . O^s_r,
//            dS = P (dO^s V^T - D_r), dQ_i += scale dS K_j, dK_j += scale dS^T Q_i,
//            dV_j += P^T dO^s_i, over the critical pairs (i, j);
//   linear:  dnum = dO^l / den, dden = -(dO^l . O^l) / den,
//            dphi(Q_i) = dnum H_i^T + dden Z_i^T, dH_i = phi(Q_i)^T dnum,
//            dZ_i = phi(Q_i)^T dden; with A_j = sum of dH_i and b_j = sum of
//            dZ_i over the rows i that have j marginal,
//            dphi(K_j) = V_j A_j^T + 1 b_j^T, dV_j += phi(K_j) A_j;
//            then the feature map's Jacobian.
// H_i and A_j are formed by complement, as in the forward: H_i = H_tot -
// sum over the excluded blocks of h_j, A_j = dH_tot - sum over the query
// blocks that exclude j of dH_i, with h_j and dH_i kept per block (d x d,
// stored in bf16 and summed in fp32: H_i and A_j enter the tensor cores in
// bf16 anyway). Every product runs on the tensor cores (mma.sync m16n8k16,
// bf16 in, fp32 accumulate); every reduction runs in a fixed order, so the
// gradients are bitwise reproducible.
#include "sla_internal.cuh"

namespace sla {
namespace {

using bf16 = __nv_bfloat16;

// Padded row-major bf16 tiles: 64 (or D) rows of D columns, row stride D + 8
// elements, so the eight rows an m16n8k16 fragment load touches fall in
// distinct banks.
template <int D>
struct Bw {
  static constexpr int LD = D + 8;
  static constexpr int kTile = 64 * LD;  // elements of a 64-row tile
  static constexpr int kMat = D * LD;    // elements of a D-row tile
  static constexpr int NT = D / 8;       // 8-column n tiles across D
};

// two consecutive elements of one row (low half = lower column)
__device__ __forceinline__ uint32_t pair_row(const bf16* t, int ld, int r, int c) {
  return *reinterpret_cast<const uint32_t*>(t + r * ld + c);
}
// one column's elements of two consecutive rows (low half = lower row)
__device__ __forceinline__ uint32_t pair_col(const bf16* t, int ld, int r, int c) {
  const uint32_t lo = *reinterpret_cast<const uint16_t*>(t + r * ld + c);
  const uint32_t hi = *reinterpret_cast<const uint16_t*>(t + (r + 1) * ld + c);
  return lo | (hi << 16);
}

// rows [0, nvalid) of a [64, D] block at src into a padded tile; the other rows zero
template <int D>
__device__ __forceinline__ void load_tile(bf16* dst, const bf16* src, int nvalid, int rows = 64) {
  constexpr int CPR = D / 8;
  for (int id = threadIdx.x; id < rows * CPR; id += blockDim.x) {
    const int r = id / CPR, ch = id % CPR;
    const bool v = r < nvalid;
    cp_async16(smem_u32(dst + r * Bw<D>::LD + ch * 8), v ? static_cast<const void*>(src + size_t(r) * D + ch * 8)
                                                           : static_cast<const void*>(src),
               v);
  }
}

// Fragments by ldmatrix from padded row-major tiles (row addresses 16-byte
// aligned: the row stride is 2 (D + 8) = 16 (D / 8 + 1) bytes).
// A: rows r0 .. r0+15, columns k0 .. k0+15
__device__ __forceinline__ void lda(uint32_t* a, const bf16* X, int ldx, int r0, int k0, int lane) {
  const int r = r0 + (lane & 7) + ((lane >> 3) & 1) * 8, c = k0 + (lane >> 4) * 8;
  ldsm_x4(smem_u32(X + r * ldx + c), a[0], a[1], a[2], a[3]);
}
// B of n tiles n0 and n0 + 8 when B[k][n] = Y[n][k] (Y rows n, k contiguous):
// b[0], b[1] for n0, b[2], b[3] for n0 + 8
__device__ __forceinline__ void ldb_rows(uint32_t* b, const bf16* Y, int ldy, int n0, int k0, int lane) {
  const int r = n0 + (lane & 7) + (lane >> 4) * 8, c = k0 + ((lane >> 3) & 1) * 8;
  ldsm_x4(smem_u32(Y + r * ldy + c), b[0], b[1], b[2], b[3]);
}
// B of n tiles n0 and n0 + 8 when B[k][n] = Z[k][n] (Z rows k, n contiguous)
__device__ __forceinline__ void ldb_cols(uint32_t* b, const bf16* Z, int ldz, int k0, int n0, int lane) {
  const int r = k0 + (lane & 7) + ((lane >> 3) & 1) * 8, c = n0 + (lane >> 4) * 8;
  ldsm_x4_t(smem_u32(Z + r * ldz + c), b[0], b[1], b[2], b[3]);
}

// acc[16 x 8 NTN] += X[r0 .. r0+15][0 .. K) * Y[0 .. 8 NTN)[0 .. K)^T
template <int NTN, int K>
__device__ __forceinline__ void mma_xyt(float (*acc)[4], const bf16* X, int ldx, int r0, const bf16* Y, int ldy,
                                        int lane) {
#pragma unroll
  for (int k0 = 0; k0 < K; k0 += 16) {
    uint32_t a[4];
    lda(a, X, ldx, r0, k0, lane);
#pragma unroll
    for (int nt = 0; nt < NTN; nt += 2) {
      uint32_t b[4];
      ldb_rows(b, Y, ldy, nt * 8, k0, lane);
      mma16816(acc[nt], a, b[0], b[1]);
      mma16816(acc[nt + 1], a, b[2], b[3]);
    }
  }
}

// acc[16 x 8 NTN] += X[r0 .. r0+15][0 .. K) * Z[0 .. K)[0 .. 8 NTN)
template <int NTN, int K>
__device__ __forceinline__ void mma_xz(float (*acc)[4], const bf16* X, int ldx, int r0, const bf16* Z, int ldz,
                                       int lane) {
#pragma unroll
  for (int k0 = 0; k0 < K; k0 += 16) {
    uint32_t a[4];
    lda(a, X, ldx, r0, k0, lane);
#pragma unroll
    for (int nt = 0; nt < NTN; nt += 2) {
      uint32_t b[4];
      ldb_cols(b, Z, ldz, k0, nt * 8, lane);
      mma16816(acc[nt], a, b[0], b[1]);
      mma16816(acc[nt + 1], a, b[2], b[3]);
    }
  }
}

// acc[16 x 8 NTN] += P * Z[0 .. 16 KT)[0 .. 8 NTN), P the 16 x 16 KT
// accumulator fragments p[2 KT][4] of an earlier product (the C layout of
// m16n8 is the A layout of the next m16n8k16)
template <int NTN, int KT>
__device__ __forceinline__ void mma_pz(float (*acc)[4], const float (*p)[4], const bf16* Z, int ldz, int lane) {
#pragma unroll
  for (int kt = 0; kt < KT; ++kt) {
    uint32_t a[4];
    a[0] = pack_bf16(p[2 * kt][0], p[2 * kt][1]);
    a[1] = pack_bf16(p[2 * kt][2], p[2 * kt][3]);
    a[2] = pack_bf16(p[2 * kt + 1][0], p[2 * kt + 1][1]);
    a[3] = pack_bf16(p[2 * kt + 1][2], p[2 * kt + 1][3]);
#pragma unroll
    for (int nt = 0; nt < NTN; nt += 2) {
      uint32_t b[4];
      ldb_cols(b, Z, ldz, kt * 16, nt * 8, lane);
      mma16816(acc[nt], a, b[0], b[1]);
      mma16816(acc[nt + 1], a, b[2], b[3]);
    }
  }
}

__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}
__device__ __forceinline__ float quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
}

// the row values of a padded tile at this lane's C-fragment positions
template <int NT>
__device__ __forceinline__ void frag_from_tile(float (*x)[4], const bf16* t, int ld, int ra, int g, int q) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const uint32_t lo = pair_row(t, ld, ra, nt * 8 + 2 * q), hi = pair_row(t, ld, ra + 8, nt * 8 + 2 * q);
    x[nt][0] = bf16_lo(lo);
    x[nt][1] = bf16_hi(lo);
    x[nt][2] = bf16_lo(hi);
    x[nt][3] = bf16_hi(hi);
  }
}

// x <- phi(x) for the two rows a lane holds (e = 0, 1: row a; 2, 3: row b);
// the four lanes of a quad hold a whole row. Softmax over the row, or elu + 1.
template <int NT>
__device__ __forceinline__ void phi_frag(float (*x)[4], bool elu1) {
  if (elu1) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) x[nt][e] = x[nt][e] > 0.0f ? x[nt][e] + 1.0f : expf(x[nt][e]);
    return;
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float m = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) m = fmaxf(m, fmaxf(x[nt][2 * h], x[nt][2 * h + 1]));
    m = quad_max(m);
    float s = 0.0f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 2 * h; e < 2 * h + 2; ++e) {
        x[nt][e] = expf(x[nt][e] - m);
        s += x[nt][e];
      }
    const float inv = 1.0f / quad_sum(s);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      x[nt][2 * h] *= inv;
      x[nt][2 * h + 1] *= inv;
    }
  }
}

// dy <- the gradient with respect to x of phi(x) . dy, from y = phi(x) alone:
// softmax y (dy - dy . y); elu + 1 dy where y > 1 (x > 0), else dy y (= dy e^x)
template <int NT>
__device__ __forceinline__ void phi_vjp_frag(float (*dy)[4], const float (*y)[4], bool elu1) {
  if (elu1) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) dy[nt][e] = y[nt][e] > 1.0f ? dy[nt][e] : dy[nt][e] * y[nt][e];
    return;
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float dot = 0.0f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) dot += dy[nt][2 * h] * y[nt][2 * h] + dy[nt][2 * h + 1] * y[nt][2 * h + 1];
    dot = quad_sum(dot);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 2 * h; e < 2 * h + 2; ++e) dy[nt][e] = y[nt][e] * (dy[nt][e] - dot);
  }
}

// rows ra, ra + 8 of a [*, D] bf16 tensor from C fragments (zero for invalid rows)
template <int NT>
__device__ __forceinline__ void store_frag_rows(bf16* dst, int D, int ra, bool va, bool vb, const float (*x)[4],
                                                int q) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int c = nt * 8 + 2 * q;
    *reinterpret_cast<uint32_t*>(dst + size_t(ra) * D + c) = va ? pack_bf16(x[nt][0], x[nt][1]) : 0u;
    *reinterpret_cast<uint32_t*>(dst + size_t(ra + 8) * D + c) = vb ? pack_bf16(x[nt][2], x[nt][3]) : 0u;
  }
}

// ---------------------------------------------------------------------------
// per-block X^T Y: out[bh][blk] = sum over the block's valid rows of x_r^T y_r
// ---------------------------------------------------------------------------
// out is float32, or bf16 for the matrices only the complement sums read
template <int D, typename OutT>
__global__ void __launch_bounds__(2 * D) block_xty_kernel(const bf16* __restrict__ X, const bf16* __restrict__ Y,
                                                          OutT* __restrict__ out, int N, int Npad, int Nb) {
  using T = Bw<D>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  bf16* Xs = reinterpret_cast<bf16*>(smem_raw);
  bf16* Ys = Xs + T::kTile;
  const int blk = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int t0 = blk * 64, nv = min(64, N - t0);
  const size_t base = (size_t(bh) * Npad + t0) * D;
  load_tile<D>(Xs, X + base, nv);
  load_tile<D>(Ys, Y + base, nv);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  const int m0 = warp * 16;  // rows of X^T = columns of X
  float acc[T::NT][4];
#pragma unroll
  for (int nt = 0; nt < T::NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
#pragma unroll
  for (int k0 = 0; k0 < 64; k0 += 16) {
    uint32_t a[4];
    a[0] = pair_col(Xs, T::LD, k0 + 2 * q, m0 + g);
    a[1] = pair_col(Xs, T::LD, k0 + 2 * q, m0 + g + 8);
    a[2] = pair_col(Xs, T::LD, k0 + 8 + 2 * q, m0 + g);
    a[3] = pair_col(Xs, T::LD, k0 + 8 + 2 * q, m0 + g + 8);
#pragma unroll
    for (int nt = 0; nt < T::NT; ++nt)
      mma16816(acc[nt], a, pair_col(Ys, T::LD, k0 + 2 * q, nt * 8 + g), pair_col(Ys, T::LD, k0 + 8 + 2 * q, nt * 8 + g));
  }
  OutT* o = out + (size_t(bh) * Nb + blk) * D * D;
#pragma unroll
  for (int nt = 0; nt < T::NT; ++nt) {
    const int c = nt * 8 + 2 * q;
    if constexpr (sizeof(OutT) == 4) {
      *reinterpret_cast<float2*>(o + (m0 + g) * D + c) = make_float2(acc[nt][0], acc[nt][1]);
      *reinterpret_cast<float2*>(o + (m0 + g + 8) * D + c) = make_float2(acc[nt][2], acc[nt][3]);
    } else {
      *reinterpret_cast<uint32_t*>(o + (m0 + g) * D + c) = pack_bf16(acc[nt][0], acc[nt][1]);
      *reinterpret_cast<uint32_t*>(o + (m0 + g + 8) * D + c) = pack_bf16(acc[nt][2], acc[nt][3]);
    }
  }
}

// out[o][e] = sum over b (ascending) of in[o][b][e], in float32
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }
template <typename InT>
__global__ void __launch_bounds__(256) reduce_blocks_kernel(const InT* __restrict__ in, float* __restrict__ out,
                                                            int nb, int E) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x, o = blockIdx.y;
  if (e >= E) return;
  const InT* p = in + size_t(o) * nb * E + e;
  float s = 0.0f;
  for (int b = 0; b < nb; ++b) s += to_f32(p[size_t(b) * E]);
  out[size_t(o) * E + e] = s;
}

// per key block j: the query blocks i with Mc[i][j] = 1 (colC) and with
// Mc[i][j] != 0 (colE), ascending
__global__ void __launch_bounds__(128) collist_kernel(const int8_t* __restrict__ Mc, int* __restrict__ colC,
                                                      int* __restrict__ colE, int* __restrict__ cntC,
                                                      int* __restrict__ cntE, int Nb) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x, bh = blockIdx.y;
  if (j >= Nb) return;
  const int8_t* m = Mc + size_t(bh) * Nb * Nb + j;
  int* lc = colC + (size_t(bh) * Nb + j) * Nb;
  int* le = colE + (size_t(bh) * Nb + j) * Nb;
  int nc = 0, ne = 0;
  for (int i = 0; i < Nb; ++i) {
    const int8_t v = m[size_t(i) * Nb];
    if (v == 1) lc[nc++] = i;
    if (v != 0) le[ne++] = i;
  }
  cntC[size_t(bh) * Nb + j] = nc;
  cntE[size_t(bh) * Nb + j] = ne;
}

// ---------------------------------------------------------------------------
// per query block: dO^l, D, dnum, dden, phi(Q), dZ_i and the alpha partial
// ---------------------------------------------------------------------------
struct PrepArgs {
  const bf16 *dO, *Os, *Ol, *Q, *W;
  const float* den;
  const float* alpha;
  bf16 *dnum, *phiq;
  float *Drow, *dden, *dzblk, *dapart;
  int B, H, N, Npad, Nb, phi_elu1;
};

template <int D, bool SLA>
__global__ void __launch_bounds__(128) bwd_prep_kernel(const PrepArgs a) {
  using T = Bw<D>;
  constexpr int NT = T::NT;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  bf16* dOs = reinterpret_cast<bf16*>(smem_raw);
  bf16* Oss = dOs + T::kTile;
  bf16* Ols = Oss + T::kTile;
  bf16* Qs = Ols + T::kTile;
  bf16* Ws = Qs + T::kTile;  // SLA: [D][LD]
  float* red = reinterpret_cast<float*>(Ws + (SLA ? T::kMat : 0));  // [4][D]
  float* ared = red + 4 * D;                                         // [4]
  const int blk = blockIdx.x, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int t0 = blk * 64, nv = min(64, a.N - t0);
  const size_t rowbase = size_t(bh) * a.Npad + t0;
  load_tile<D>(dOs, a.dO + rowbase * D, nv);
  load_tile<D>(Oss, a.Os + rowbase * D, nv);
  load_tile<D>(Ols, a.Ol + rowbase * D, nv);
  load_tile<D>(Qs, a.Q + rowbase * D, nv);
  if (SLA && a.W != nullptr) load_tile<D>(Ws, a.W, D, D);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  const int ra = warp * 16 + g, rb = ra + 8;
  const bool va = ra < nv, vb = rb < nv;
  const float alpha = SLA ? 1.0f : a.alpha[h];
  // dO^l: SLA dO W^T (y = x W; dO without W), SLA2 (1 - alpha) dO
  float u[NT][4];
  if (SLA && a.W != nullptr) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) u[nt][0] = u[nt][1] = u[nt][2] = u[nt][3] = 0.0f;
    mma_xyt<NT, D>(u, dOs, T::LD, warp * 16, Ws, T::LD, lane);
  } else {  // SLA without W (identity) or SLA2
    frag_from_tile<NT>(u, dOs, T::LD, ra, g, q);
    const float lmul = SLA ? 1.0f : 1.0f - alpha;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) u[nt][e] *= lmul;
  }
  float x[NT][4], y[NT][4];
  // D_r = dO^s . O^s and the alpha partial sum(dO (O^s - O^l))
  frag_from_tile<NT>(x, dOs, T::LD, ra, g, q);
  frag_from_tile<NT>(y, Oss, T::LD, ra, g, q);
  float Da = 0.0f, Db = 0.0f, ap = 0.0f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    Da += x[nt][0] * y[nt][0] + x[nt][1] * y[nt][1];
    Db += x[nt][2] * y[nt][2] + x[nt][3] * y[nt][3];
  }
  frag_from_tile<NT>(y, Ols, T::LD, ra, g, q);
  if constexpr (!SLA) {
    float sa = 0.0f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sa += x[nt][e] * y[nt][e];
    ap = (Da + Db) - sa;  // this lane's dO . (O^s - O^l)
  }
  Da = quad_sum(Da) * alpha;
  Db = quad_sum(Db) * alpha;
  // dden = -(dO^l . O^l) / den, dnum = dO^l / den (0 without a marginal block)
  float ea = 0.0f, eb = 0.0f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    ea += u[nt][0] * y[nt][0] + u[nt][1] * y[nt][1];
    eb += u[nt][2] * y[nt][2] + u[nt][3] * y[nt][3];
  }
  ea = quad_sum(ea);
  eb = quad_sum(eb);
  const float dena = va ? a.den[rowbase + ra] : 0.0f, denb = vb ? a.den[rowbase + rb] : 0.0f;
  const float ia = dena != 0.0f ? 1.0f / dena : 0.0f, ib = denb != 0.0f ? 1.0f / denb : 0.0f;
  const float dda = -ea * ia, ddb = -eb * ib;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    u[nt][0] *= ia;
    u[nt][1] *= ia;
    u[nt][2] *= ib;
    u[nt][3] *= ib;
  }
  store_frag_rows<NT>(a.dnum + rowbase * D, D, ra, va, vb, u, q);
  // phi(Q) rows (zero past N) and dZ_i = sum_r dden_r phi(q_r)
  frag_from_tile<NT>(y, Qs, T::LD, ra, g, q);
  phi_frag<NT>(y, a.phi_elu1 != 0);
  store_frag_rows<NT>(a.phiq + rowbase * D, D, ra, va, vb, y, q);
  if (q == 0) {
    if (va) {
      a.Drow[rowbase + ra] = Da;
      a.dden[rowbase + ra] = dda;
    }
    if (vb) {
      a.Drow[rowbase + rb] = Db;
      a.dden[rowbase + rb] = ddb;
    }
  }
  const float wa = va ? dda : 0.0f, wb = vb ? ddb : 0.0f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float z = wa * y[nt][e] + wb * y[nt][2 + e];
      z += __shfl_xor_sync(0xffffffffu, z, 4);
      z += __shfl_xor_sync(0xffffffffu, z, 8);
      z += __shfl_xor_sync(0xffffffffu, z, 16);
      if (g == 0) red[warp * D + nt * 8 + 2 * q + e] = z;
    }
  if constexpr (!SLA) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ap += __shfl_xor_sync(0xffffffffu, ap, off);
    if (lane == 0) ared[warp] = ap;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += 128)
    a.dzblk[(size_t(bh) * a.Nb + blk) * D + c] = ((red[c] + red[D + c]) + red[2 * D + c]) + red[3 * D + c];
  if constexpr (!SLA) {
    if (threadIdx.x == 0) a.dapart[(size_t(h) * a.B + b) * a.Nb + blk] = ((ared[0] + ared[1]) + ared[2]) + ared[3];
  }
}

// dst (bf16 [D][LD] tile) = tot - sum over the listed blocks of blk[j] (bf16
// d x d each, summed in fp32), and zdst[c] = ztot[c] - sum of zblk[j][c]: the complement sums
// of H_i, Z_i (query side) and A_j, b_j (key side). Each of the NTH threads
// keeps its D * D / NTH entries in registers and subtracts block after block (coalesced
// float4 loads, independent across the thread's entries), in list order.
template <int D, int NTH>
__device__ __forceinline__ void complement_sum(bf16* dst, float* zdst, const float* tot, const bf16* blk,
                                               const float* ztot, const float* zblk, const int32_t* l1, int n1,
                                               const int32_t* l2, int n2) {
  constexpr int PER = D * D / 4 / NTH;
  const int tid = threadIdx.x;
  float4 acc[PER];
  const float4* t4 = reinterpret_cast<const float4*>(tot);
#pragma unroll
  for (int k = 0; k < PER; ++k) acc[k] = t4[tid + NTH * k];
  float z = tid < D ? ztot[tid] : 0.0f;
  auto sub = [&](int j) {
    const uint2* b4 = reinterpret_cast<const uint2*>(blk + size_t(j) * D * D);  // 4 bf16 per load
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const uint2 v = b4[tid + NTH * k];
      acc[k].x -= bf16_lo(v.x);
      acc[k].y -= bf16_hi(v.x);
      acc[k].z -= bf16_lo(v.y);
      acc[k].w -= bf16_hi(v.y);
    }
    if (tid < D) z -= zblk[size_t(j) * D + tid];
  };
  for (int u = 0; u < n1; ++u) sub(l1[u]);
  for (int u = 0; u < n2; ++u) sub(l2[u]);
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int e = 4 * (tid + NTH * k), r = e / D, c = e % D;
    *reinterpret_cast<uint2*>(dst + r * Bw<D>::LD + c) =
        make_uint2(pack_bf16(acc[k].x, acc[k].y), pack_bf16(acc[k].z, acc[k].w));
  }
  if (tid < D) zdst[tid] = z;
}

// ---------------------------------------------------------------------------
// dQ per query block: the sparse pairs, then the linear branch
// ---------------------------------------------------------------------------
struct QArgs {
  const bf16 *Q, *K, *V, *dO, *dnum;
  const int32_t *crit, *neg;
  const float *lse, *Drow, *dden, *htot;
  const bf16* hblk;
  const float *ztot, *zblk;
  const float* alpha;  // SLA2 [H] (dO^s = alpha dO); null for SLA
  const float* dQs;    // tcgen05 sparse partial (scaled); null: run the sparse loop here
  bf16* dQ;
  float scale, scale_log2;
  int H, N, Npad, Nb, kc, kn, phi_elu1;
};

// 8 warps: warp w takes rows 16 (w & 3) .. + 15 of the query block and keys
// 32 (w >> 2) .. + 31 of each critical key block; the two key halves' partial
// dQ are summed through shared memory, then the first half's warps add the
// linear branch and store.
template <int D>
__global__ void __launch_bounds__(256, 1) bwd_q_kernel(const QArgs a) {
  using T = Bw<D>;
  constexpr int NT = T::NT;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  bf16* Qs = reinterpret_cast<bf16*>(smem_raw);
  bf16* dOs = Qs + T::kTile;
  bf16* dns = dOs + T::kTile;  // dnum tile
  bf16* KVs = dns + T::kTile;  // [2 buffers][K tile, V tile]; after the loop: dQ partials
  bf16* Hs = KVs + 4 * T::kTile;  // [D][LD]: H_i
  float* zis = reinterpret_cast<float*>(Hs + T::kMat);  // [D]: Z_i
  const int i = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int rg = warp & 3, kh = warp >> 2;  // row group, key half
  const int t0 = i * 64, nv = min(64, a.N - t0);
  const float asc = a.alpha ? a.alpha[bh % a.H] : 1.0f;  // dO^s = asc dO
  const bool linear = a.kc + a.kn < a.Nb;
  const size_t rowbase = size_t(bh) * a.Npad + t0;
  const size_t headbase = size_t(bh) * a.Npad * D;
  const int32_t* crit = a.crit + (size_t(bh) * a.Nb + i) * a.kc;
  load_tile<D>(Qs, a.Q + rowbase * D, nv);
  load_tile<D>(dOs, a.dO + rowbase * D, nv);
  if (linear) load_tile<D>(dns, a.dnum + rowbase * D, nv);
  cp_async_commit();
  auto load_pair = [&](int t) {
    const int j = crit[t];
    const int nvj = min(64, a.N - j * 64);
    bf16* buf = KVs + (t & 1) * 2 * T::kTile;
    load_tile<D>(buf, a.K + headbase + size_t(j) * 64 * D, nvj);
    load_tile<D>(buf + T::kTile, a.V + headbase + size_t(j) * 64 * D, nvj);
    cp_async_commit();
  };
  if (!a.dQs) load_pair(0);
  // H_i = H_tot - sum over the excluded blocks of h_j, Z_i likewise (while the
  // first tiles land)
  if (linear)
    complement_sum<D, 256>(Hs, zis, a.htot + size_t(bh) * D * D, a.hblk + size_t(bh) * a.Nb * D * D,
                           a.ztot + size_t(bh) * D, a.zblk + size_t(bh) * a.Nb * D, crit, a.kc,
                           a.neg + (size_t(bh) * a.Nb + i) * a.kn, a.kn);

  const int r0 = rg * 16, ra = r0 + g, rb = ra + 8;
  const bool va = ra < nv, vb = rb < nv;
  const float lse2a = va ? a.lse[rowbase + ra] * kLog2e : INFINITY;
  const float lse2b = vb ? a.lse[rowbase + rb] * kLog2e : INFINITY;
  const float Da = va ? a.Drow[rowbase + ra] : 0.0f, Db = vb ? a.Drow[rowbase + rb] : 0.0f;

  float dq[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) dq[nt][0] = dq[nt][1] = dq[nt][2] = dq[nt][3] = 0.0f;
  const int nsteps = a.dQs ? 0 : a.kc;
  for (int t = 0; t < nsteps; ++t) {
    if (t + 1 < nsteps) {
      load_pair(t + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const bf16* Ks = KVs + (t & 1) * 2 * T::kTile + kh * 32 * T::LD;  // this warp's 32 keys
    const bf16* Vs = Ks + T::kTile;
    const int nvj = min(64, a.N - crit[t] * 64) - kh * 32;
    float s[4][4], dp[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.0f;
    mma_xyt<4, D>(s, Qs, T::LD, r0, Ks, T::LD, lane);
    mma_xyt<4, D>(dp, dOs, T::LD, r0, Vs, T::LD, lane);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = nt * 8 + 2 * q + (e & 1);
        const float p = key < nvj ? ex2_approx(fmaf(s[nt][e], a.scale_log2, -(e < 2 ? lse2a : lse2b))) : 0.0f;
        s[nt][e] = p * (asc * dp[nt][e] - (e < 2 ? Da : Db));  // dS
      }
    mma_pz<NT, 2>(dq, s, Ks, T::LD, lane);
    __syncthreads();  // this buffer is refilled two pairs on
  }
  cp_async_wait<0>();  // Q, dO, dnum landed even without a sparse pair (the barrier below publishes them)
  // the two key halves' partial dQ: the second half's warps hand theirs over
  // (rows D + 4 floats apart, so a fragment's eight rows fall in distinct banks)
  constexpr int RS = D + 4;
  float* red = reinterpret_cast<float*>(KVs);  // [64 rows][RS]
  if (kh == 1) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c = nt * 8 + 2 * q;
      *reinterpret_cast<float2*>(red + (r0 + g) * RS + c) = make_float2(dq[nt][0], dq[nt][1]);
      *reinterpret_cast<float2*>(red + (r0 + g + 8) * RS + c) = make_float2(dq[nt][2], dq[nt][3]);
    }
  }
  __syncthreads();
  if (kh == 1) return;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int c = nt * 8 + 2 * q;
    const float2 x0 = *reinterpret_cast<const float2*>(red + (r0 + g) * RS + c);
    const float2 x1 = *reinterpret_cast<const float2*>(red + (r0 + g + 8) * RS + c);
    dq[nt][0] = (dq[nt][0] + x0.x) * a.scale;
    dq[nt][1] = (dq[nt][1] + x0.y) * a.scale;
    dq[nt][2] = (dq[nt][2] + x1.x) * a.scale;
    dq[nt][3] = (dq[nt][3] + x1.y) * a.scale;
  }
  if (a.dQs) {  // the tcgen05 loop's partial (already scaled)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c = nt * 8 + 2 * q;
      if (va) {
        const float2 x = *reinterpret_cast<const float2*>(a.dQs + (rowbase + ra) * D + c);
        dq[nt][0] += x.x;
        dq[nt][1] += x.y;
      }
      if (vb) {
        const float2 x = *reinterpret_cast<const float2*>(a.dQs + (rowbase + rb) * D + c);
        dq[nt][2] += x.x;
        dq[nt][3] += x.y;
      }
    }
  }

  if (linear) {
    // dphi(Q_i) = dnum H_i^T + dden Z_i^T, through the feature map's Jacobian
    float u[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) u[nt][0] = u[nt][1] = u[nt][2] = u[nt][3] = 0.0f;
    mma_xyt<NT, D>(u, dns, T::LD, r0, Hs, T::LD, lane);
    const float dda = va ? a.dden[rowbase + ra] : 0.0f, ddb = vb ? a.dden[rowbase + rb] : 0.0f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c = nt * 8 + 2 * q;
      u[nt][0] += dda * zis[c];
      u[nt][1] += dda * zis[c + 1];
      u[nt][2] += ddb * zis[c];
      u[nt][3] += ddb * zis[c + 1];
    }
    float y[NT][4];
    frag_from_tile<NT>(y, Qs, T::LD, ra, g, q);
    phi_frag<NT>(y, a.phi_elu1 != 0);
    phi_vjp_frag<NT>(u, y, a.phi_elu1 != 0);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) dq[nt][e] += u[nt][e];
  }
  store_frag_rows<NT>(a.dQ + rowbase * D, D, ra, va, vb, dq, q);
}

// ---------------------------------------------------------------------------
// dK, dV per key block: the sparse pairs (query blocks with this block
// critical), then the linear branch
// ---------------------------------------------------------------------------
struct KVArgs {
  const bf16 *Q, *K, *V, *dO, *phik;
  const int *colC, *colE, *cntC, *cntE;
  const float *lse, *Drow, *dhtot;
  const bf16* dhblk;
  const float *dztot, *dzblk;
  const float* alpha;  // SLA2 [H]; null for SLA
  const float *dKs, *dVs;  // tcgen05 sparse partials (scaled); null: run the sparse loop here
  bf16 *dK, *dV;
  float scale, scale_log2;
  int H, N, Npad, Nb, linear, phi_elu1;
};

// 8 warps: warp w takes key rows 16 (w & 3) .. + 15 of the key block and
// queries 32 (w >> 2) .. + 31 of each query block; the two query halves'
// partial dK and dV are summed through shared memory, then the first half's
// warps add the linear branch and store.
template <int D>
__global__ void __launch_bounds__(256, 1) bwd_kv_kernel(const KVArgs a) {
  using T = Bw<D>;
  constexpr int NT = T::NT;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  bf16* Ks = reinterpret_cast<bf16*>(smem_raw);
  bf16* Vs = Ks + T::kTile;
  bf16* PKs = Vs + T::kTile;
  bf16* QOs = PKs + T::kTile;     // [2 buffers][Q tile, dO tile]; after the loop: dK, dV partials
  bf16* As = QOs + 4 * T::kTile;  // [D][LD]: A_j
  float* bjs = reinterpret_cast<float*>(As + T::kMat);  // [D]
  float* lse2s = bjs + D;                               // [2][64]
  float* Ds = lse2s + 128;                              // [2][64]
  const int j = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int rg = warp & 3, qh = warp >> 2;  // key-row group, query half
  const int t0 = j * 64, nvj = min(64, a.N - t0);
  const float asc = a.alpha ? a.alpha[bh % a.H] : 1.0f;  // dO^s = asc dO
  const size_t rowbase = size_t(bh) * a.Npad + t0;
  const size_t headrow = size_t(bh) * a.Npad;
  load_tile<D>(Ks, a.K + rowbase * D, nvj);
  load_tile<D>(Vs, a.V + rowbase * D, nvj);
  load_tile<D>(PKs, a.phik + rowbase * D, nvj);
  cp_async_commit();
  const int nC = a.dKs ? 0 : a.cntC[size_t(bh) * a.Nb + j];
  const int* colC = a.colC + (size_t(bh) * a.Nb + j) * a.Nb;
  auto load_pair = [&](int t) {
    const int i = colC[t];
    const int nvi = min(64, a.N - i * 64);
    const int b = t & 1;
    bf16* buf = QOs + b * 2 * T::kTile;
    load_tile<D>(buf, a.Q + (headrow + size_t(i) * 64) * D, nvi);
    load_tile<D>(buf + T::kTile, a.dO + (headrow + size_t(i) * 64) * D, nvi);
    cp_async_commit();
    if (threadIdx.x < 64) {
      const int r = threadIdx.x;
      lse2s[b * 64 + r] = r < nvi ? a.lse[headrow + i * 64 + r] * kLog2e : INFINITY;
      Ds[b * 64 + r] = r < nvi ? a.Drow[headrow + i * 64 + r] : 0.0f;
    }
  };
  if (nC > 0) load_pair(0);
  // A_j = dH_tot - sum over the query blocks that exclude j of dH_i, b_j likewise
  if (a.linear) {
    const int nE = a.cntE[size_t(bh) * a.Nb + j];
    complement_sum<D, 256>(As, bjs, a.dhtot + size_t(bh) * D * D, a.dhblk + size_t(bh) * a.Nb * D * D,
                           a.dztot + size_t(bh) * D, a.dzblk + size_t(bh) * a.Nb * D,
                           a.colE + (size_t(bh) * a.Nb + j) * a.Nb, nE, nullptr, 0);
  }
  const int r0 = rg * 16, ra = r0 + g, rb = ra + 8;
  const bool va = ra < nvj, vb = rb < nvj;

  float dk[NT][4], dv[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[nt][e] = dv[nt][e] = 0.0f;
  for (int t = 0; t < nC; ++t) {
    if (t + 1 < nC) {
      load_pair(t + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const bf16* Qs = QOs + (t & 1) * 2 * T::kTile + qh * 32 * T::LD;  // this warp's 32 queries
    const bf16* dOs = Qs + T::kTile;
    const float* l2 = lse2s + (t & 1) * 64 + qh * 32;
    const float* Dc = Ds + (t & 1) * 64 + qh * 32;
    float st[4][4], dpt[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[nt][e] = dpt[nt][e] = 0.0f;
    mma_xyt<4, D>(st, Ks, T::LD, r0, Qs, T::LD, lane);    // S^T = K_j Q_i^T
    mma_xyt<4, D>(dpt, Vs, T::LD, r0, dOs, T::LD, lane);  // dP^T = V_j dO_i^T
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nt * 8 + 2 * q + (e & 1);
        const bool vk = e < 2 ? va : vb;
        st[nt][e] = vk ? ex2_approx(fmaf(st[nt][e], a.scale_log2, -l2[col])) : 0.0f;  // P^T
      }
    mma_pz<NT, 2>(dv, st, dOs, T::LD, lane);  // dV += P^T dO_i
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nt * 8 + 2 * q + (e & 1);
        st[nt][e] *= asc * dpt[nt][e] - Dc[col];  // dS^T
      }
    mma_pz<NT, 2>(dk, st, Qs, T::LD, lane);  // dK += dS^T Q_i
    __syncthreads();  // this buffer is refilled two pairs on
  }
  cp_async_wait<0>();
  __syncthreads();  // K, V, phi(K) and A_j are in place even without a sparse pair
  // the two query halves' partials: the second half's warps hand theirs over
  // (rows D + 4 floats apart, so a fragment's eight rows fall in distinct banks)
  constexpr int RS = D + 4;
  float* redk = reinterpret_cast<float*>(QOs);  // [64 rows][RS]
  float* redv = redk + 64 * RS;
  if (qh == 1) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c = nt * 8 + 2 * q;
      *reinterpret_cast<float2*>(redk + (r0 + g) * RS + c) = make_float2(dk[nt][0], dk[nt][1]);
      *reinterpret_cast<float2*>(redk + (r0 + g + 8) * RS + c) = make_float2(dk[nt][2], dk[nt][3]);
      *reinterpret_cast<float2*>(redv + (r0 + g) * RS + c) = make_float2(dv[nt][0], dv[nt][1]);
      *reinterpret_cast<float2*>(redv + (r0 + g + 8) * RS + c) = make_float2(dv[nt][2], dv[nt][3]);
    }
  }
  __syncthreads();
  if (qh == 1) return;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int c = nt * 8 + 2 * q;
    const float2 k0 = *reinterpret_cast<const float2*>(redk + (r0 + g) * RS + c);
    const float2 k1 = *reinterpret_cast<const float2*>(redk + (r0 + g + 8) * RS + c);
    const float2 v0 = *reinterpret_cast<const float2*>(redv + (r0 + g) * RS + c);
    const float2 v1 = *reinterpret_cast<const float2*>(redv + (r0 + g + 8) * RS + c);
    dk[nt][0] = (dk[nt][0] + k0.x) * a.scale;
    dk[nt][1] = (dk[nt][1] + k0.y) * a.scale;
    dk[nt][2] = (dk[nt][2] + k1.x) * a.scale;
    dk[nt][3] = (dk[nt][3] + k1.y) * a.scale;
    dv[nt][0] = (dv[nt][0] + v0.x) * asc;
    dv[nt][1] = (dv[nt][1] + v0.y) * asc;
    dv[nt][2] = (dv[nt][2] + v1.x) * asc;
    dv[nt][3] = (dv[nt][3] + v1.y) * asc;
  }
  if (a.dKs) {  // the sparse partials of the tcgen05 loop (already scaled); pad rows hold no data
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c = nt * 8 + 2 * q;
      if (va) {
        const float2 k0 = *reinterpret_cast<const float2*>(a.dKs + (rowbase + ra) * D + c);
        const float2 v0 = *reinterpret_cast<const float2*>(a.dVs + (rowbase + ra) * D + c);
        dk[nt][0] += k0.x; dk[nt][1] += k0.y; dv[nt][0] += v0.x; dv[nt][1] += v0.y;
      }
      if (vb) {
        const float2 k1 = *reinterpret_cast<const float2*>(a.dKs + (rowbase + rb) * D + c);
        const float2 v1 = *reinterpret_cast<const float2*>(a.dVs + (rowbase + rb) * D + c);
        dk[nt][2] += k1.x; dk[nt][3] += k1.y; dv[nt][2] += v1.x; dv[nt][3] += v1.y;
      }
    }
  }

  if (a.linear) {
    mma_xz<NT, D>(dv, PKs, T::LD, r0, As, T::LD, lane);  // dV += phi(K_j) A_j
    store_frag_rows<NT>(a.dV + rowbase * D, D, ra, va, vb, dv, q);
    float u[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) u[nt][0] = u[nt][1] = u[nt][2] = u[nt][3] = 0.0f;
    mma_xyt<NT, D>(u, Vs, T::LD, r0, As, T::LD, lane);  // V_j A_j^T
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c = nt * 8 + 2 * q;
      u[nt][0] += bjs[c];
      u[nt][1] += bjs[c + 1];
      u[nt][2] += bjs[c];
      u[nt][3] += bjs[c + 1];
    }
    float y[NT][4];
    frag_from_tile<NT>(y, Ks, T::LD, ra, g, q);
    phi_frag<NT>(y, a.phi_elu1 != 0);
    phi_vjp_frag<NT>(u, y, a.phi_elu1 != 0);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) dk[nt][e] += u[nt][e];
  } else {
    store_frag_rows<NT>(a.dV + rowbase * D, D, ra, va, vb, dv, q);
  }
  store_frag_rows<NT>(a.dK + rowbase * D, D, ra, va, vb, dk, q);
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int D>
cudaError_t run_backward(const BwdArgs& a, cudaStream_t s) {
  using T = Bw<D>;
  const BwLayout& L = a.L;
  const int BH = L.BH, Nb = L.Nb;
  const dim3 blocks(Nb, BH);
  cudaError_t e = cudaSuccess;
  // 1. dO^l, D, dnum, dden, phi(Q), dZ_i, alpha partials
  {
    PrepArgs p{a.dO, a.save_os, a.save_ol, a.Q, a.w_proj, a.save_den, a.alpha, a.dnum, a.phiq, a.Drow, a.dden,
               a.dzblk, a.dapart, L.B, L.H, L.N, L.Npad, Nb, a.phi_elu1};
    const int bytes = (4 * T::kTile + (a.sla ? T::kMat : 0)) * 2 + (4 * D + 4) * 4;
    if (a.sla) {
      e = set_smem(bwd_prep_kernel<D, true>, bytes);
      if (e == cudaSuccess) bwd_prep_kernel<D, true><<<blocks, 128, bytes, s>>>(p);
    } else {
      e = set_smem(bwd_prep_kernel<D, false>, bytes);
      if (e == cudaSuccess) bwd_prep_kernel<D, false><<<blocks, 128, bytes, s>>>(p);
    }
  }
  // 2. column lists of the mask
  if (e == cudaSuccess) {
    collist_kernel<<<dim3((Nb + 127) / 128, BH), 128, 0, s>>>(a.mc, a.colC, a.colE, a.cntC, a.cntE, Nb);
    e = cudaGetLastError();
  }
  const int xty_bytes = 2 * T::kTile * 2;
  if (e == cudaSuccess) e = set_smem(block_xty_kernel<D, bf16>, xty_bytes);
  if (e == cudaSuccess) e = set_smem(block_xty_kernel<D, float>, xty_bytes);
  if (e == cudaSuccess && L.linear) {
    // 3. h_j = phi(K_j)^T V_j and dH_i = phi(Q_i)^T dnum_i per block, their head totals
    block_xty_kernel<D, bf16><<<blocks, 2 * D, xty_bytes, s>>>(a.phik, a.V, a.hblk, L.N, L.Npad, Nb);
    block_xty_kernel<D, bf16><<<blocks, 2 * D, xty_bytes, s>>>(a.phiq, a.dnum, a.dhblk, L.N, L.Npad, Nb);
    reduce_blocks_kernel<bf16><<<dim3((D * D + 255) / 256, BH), 256, 0, s>>>(a.dhblk, a.dhtot, Nb, D * D);
    reduce_blocks_kernel<float><<<dim3((D + 255) / 256, BH), 256, 0, s>>>(a.dzblk, a.dztot, Nb, D);
    e = cudaGetLastError();
  }
  // 4. dW = sum over rows of O^l^T dO (SLA), dalpha_h = sum of the partials (SLA2)
  if (e == cudaSuccess && a.dW != nullptr) {
    block_xty_kernel<D, float><<<blocks, 2 * D, xty_bytes, s>>>(a.save_ol, a.dO, a.dwpart, L.N, L.Npad, Nb);
    reduce_blocks_kernel<float><<<dim3((D * D + 255) / 256, 1), 256, 0, s>>>(a.dwpart, a.dW, BH * Nb, D * D);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess && a.dalpha != nullptr) {
    reduce_blocks_kernel<float><<<dim3(1, L.H), 256, 0, s>>>(a.dapart, a.dalpha, L.B * Nb, 1);
    e = cudaGetLastError();
  }
  const float scale = a.scale;
  const float* alpha = a.sla ? nullptr : a.alpha;
  // 5. dQ: at d = 128 the sparse loop on tcgen05 first (fp32 partial)
  const bool tcq = D == 128 && a.dqs != nullptr;
  if (e == cudaSuccess && tcq) {
    QTcArgs ta{a.crit, a.save_lse, a.Drow, alpha, a.dqs, a.status, L.H, L.N, L.Npad, Nb, L.kc, scale,
               scale * kLog2e};
    e = launch_bwd_q_tc(a.Q, a.K, a.V, a.dO, ta, BH, s);
  }
  if (e == cudaSuccess) {
    QArgs qa{a.Q, a.K, a.V, a.dO, a.dnum, a.crit, a.neg, a.save_lse, a.Drow, a.dden, a.htot, a.hblk, a.ztot,
             a.zblk, alpha, tcq ? a.dqs : nullptr, a.dQ, scale, scale * kLog2e, L.H, L.N, L.Npad, Nb, L.kc, L.kn,
             a.phi_elu1};
    const int bytes = (7 * T::kTile + T::kMat) * 2 + D * 4;
    e = set_smem(bwd_q_kernel<D>, bytes);
    if (e == cudaSuccess) {
      bwd_q_kernel<D><<<blocks, 256, bytes, s>>>(qa);
      e = cudaGetLastError();
    }
  }
  // 6. dK, dV: at d = 128 the sparse loop on tcgen05 first (fp32 partials)
  // (the lse rows arrive by bulk copy: 16-byte aligned global addresses only)
  const bool tc = D == 128 && a.dks != nullptr && (reinterpret_cast<uintptr_t>(a.save_lse) & 15) == 0;
  if (e == cudaSuccess && tc) {
    KvTcArgs ta{a.colC, a.cntC, a.save_lse, a.Drow, alpha, a.dks, a.dvs, a.status, L.H, L.N, L.Npad, Nb, scale,
                scale * kLog2e};
    e = launch_bwd_kv_tc(a.Q, a.K, a.V, a.dO, ta, BH, s);
  }
  if (e == cudaSuccess) {
    KVArgs ka{a.Q, a.K, a.V, a.dO, a.phik, a.colC, a.colE, a.cntC, a.cntE, a.save_lse, a.Drow, a.dhtot,
              a.dhblk, a.dztot, a.dzblk, alpha, tc ? a.dks : nullptr, tc ? a.dvs : nullptr, a.dK, a.dV, scale,
              scale * kLog2e, L.H, L.N, L.Npad, Nb, L.linear ? 1 : 0, a.phi_elu1};
    const int bytes = (7 * T::kTile + T::kMat) * 2 + (D + 256) * 4;
    e = set_smem(bwd_kv_kernel<D>, bytes);
    if (e == cudaSuccess) {
      bwd_kv_kernel<D><<<blocks, 256, bytes, s>>>(ka);
      e = cudaGetLastError();
    }
  }
  return e;
}

}  // namespace

cudaError_t launch_backward(const BwdArgs& a, cudaStream_t s) {
  return a.L.d == 128 ? run_backward<128>(a, s) : run_backward<64>(a, s);
}

}  // namespace sla
