// Steps 1 and 3 of the forward as two streaming passes over the inputs (bf16,
// d = 128): every 64-token block of Q, K and V is read from HBM once.
//
//   q_stream_kernel:  qbar_i = mean of Q's block i (valid rows; SLA2: times
//                     proj_q) and, when the linear branch takes phi(Q)
//                     precomputed, the phi(Q) rows.
//   kv_stream_kernel: kbar_j = mean of K's block j (SLA2: times proj_k), the
//                     phi(K) rows, z_j = sum of block j's phi(K) rows, and the
//                     chunk's partial H = sum_j phi(K_j)^T V_j (tcgen05) and Z.
//
// Sources: SLA structured summary (aipaper.cc), section 4, formula 1 (pool =
// average over each block of the sequence) and formula 3 (H_i, Z_i);
// SLA walkthrough (intelliparadigm.com), section 1.2 (precompute
// h_j = phi(K_j)^T V_j, z_j = rowsum(phi(K_j)^T)) and section 3.2 (phi =
// softmax over the head dimension); SLA2 notes (zhaifeiyue.github.io),
// section 2, and SLA2 article (mcffsbgs.com): the router's proj_q / proj_k.
//
// The pooled vectors follow the same fixed float32 order as the mask path
// everywhere (ascending sums from +0, products and sums rounded separately),
// so the mask they rank is reproducible bit for bit.
//
// Layout: one CTA per (chunk of consecutive blocks, head), chunks sized so
// that the grid is about two CTAs per SM of a 148-SM B200 (the partial sums
// of a chunk are added in a fixed order afterwards). Warp 4 streams 64 x 64
// bf16 boxes by TMA into a ring of shared-memory stages (128-byte swizzle,
// rows past N zero-filled); warps 0-3 compute; in kv_stream_kernel warp 5
// issues the tcgen05 products into a 128-column TMEM accumulator. The phi
// rows are written back over the input tile they were computed from, and
// leave through TMA stores from there, so the whole shared memory serves the
// ring: two blocks stay in flight per CTA while a third is computed. Every
// wait is bounded.
#include <string.h>

#include "tc_util.cuh"

namespace sla {

using namespace tc;

namespace {

constexpr int SD = 128;                // head dimension of these kernels
constexpr int kSub = 64 * 128;         // one 64-row x 128-byte SW128 box (64 bf16 columns)
constexpr int kTileBytes = 2 * kSub;   // a 64 x 128 bf16 block tile
constexpr int kQStages = 4, kKvStages = 3;

// byte offset of element (t, c) of a block tile (two SW128 boxes)
__device__ __forceinline__ uint32_t elem_off(int t, int c) {
  return uint32_t(c >> 6) * kSub + uint32_t(t) * 128u + (uint32_t(((c & 63) >> 3) ^ (t & 7)) << 4) +
         (uint32_t(c & 7) << 1);
}
// byte offset of 16-byte chunk q (columns 64 h + 8 q .. + 7) of row t
__device__ __forceinline__ uint32_t chunk_off(int h, int t, int q) {
  return uint32_t(h) * kSub + uint32_t(t) * 128u + (uint32_t(q ^ (t & 7)) << 4);
}

// Byte offsets of column c in rows 0..7 of a block tile; row t's offset is
// colo[t & 7] + (t & ~7) * 128 (the swizzle pattern repeats every 8 rows).
__device__ __forceinline__ void column_offsets(int c, uint32_t (&colo)[8]) {
#pragma unroll
  for (int t = 0; t < 8; ++t) colo[t] = elem_off(t, c);
}
__device__ __forceinline__ float elem_at(const unsigned char* tile, const uint32_t (&colo)[8], int t) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + colo[t & 7] + (t & ~7) * 128));
}

// Column c of a block tile summed over rows 0..n-1 in ascending order from +0,
// then the mean: times 2^-6 for a full block, one rounded division otherwise.
__device__ __forceinline__ float pool_column(const unsigned char* tile, const uint32_t (&colo)[8], int c, int n) {
  float acc = 0.0f;
  if (n == kBlock) {
#pragma unroll
    for (int t = 0; t < kBlock; ++t) acc = __fadd_rn(acc, elem_at(tile, colo, t));
    return __fmul_rn(acc, 0.015625f);
  }
  // the partial last block of a sequence
  for (int t = 0; t < n; ++t)
    acc = __fadd_rn(acc, __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + elem_off(t, c))));
  return __fdiv_rn(acc, float(n));
}

// The router projection of up to kRouterBatch pooled rows at once (SLA2):
// out[r][c] = sum_k x[r][k] W[k][c], k ascending, products rounded
// separately. Thread c loads W[k][c] once per k for the whole batch, so the
// weight loads are amortised over the batch's rows.
constexpr int kRouterBatch = 16;
__device__ __forceinline__ void router_batch(const float (*x)[SD], int rows, const __nv_bfloat16* __restrict__ W,
                                             int c, float* out_base, size_t out_stride) {
  float acc[kRouterBatch];
#pragma unroll
  for (int r = 0; r < kRouterBatch; ++r) acc[r] = 0.0f;
  // 16 weights in flight at a time, then their products for every row
#pragma unroll 1
  for (int k0 = 0; k0 < SD; k0 += 16) {
    float w[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) w[u] = __bfloat162float(__ldg(W + (k0 + u) * SD + c));
#pragma unroll
    for (int r = 0; r < kRouterBatch; ++r) {
      if (r < rows) {
#pragma unroll
        for (int u4 = 0; u4 < 4; ++u4) {
          const float4 xv = *reinterpret_cast<const float4*>(&x[r][k0 + 4 * u4]);
          acc[r] = __fadd_rn(acc[r], __fmul_rn(xv.x, w[4 * u4]));
          acc[r] = __fadd_rn(acc[r], __fmul_rn(xv.y, w[4 * u4 + 1]));
          acc[r] = __fadd_rn(acc[r], __fmul_rn(xv.z, w[4 * u4 + 2]));
          acc[r] = __fadd_rn(acc[r], __fmul_rn(xv.w, w[4 * u4 + 3]));
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRouterBatch; ++r)
    if (r < rows) out_base[r * out_stride + c] = acc[r];
}

// phi of one row, computed by two threads (half h of the row each: its 64
// columns are sub-tile h of the row): softmax over the 128 values, or elu + 1
// elementwise. xmax / xsum exchange the halves' partial max / sum through
// shared memory; `bar` is the 128-thread named barrier of the compute warps.
// Rows t >= n (past N) become zero. The row's 64 values of half h are
// returned packed as bf16 pairs in out[32].
__device__ __forceinline__ void phi_row_half(const unsigned char* tile, const uint32_t (&rowo)[8], int t, int h,
                                             int n, bool elu1, float (*xmax)[64], float (*xsum)[64],
                                             uint32_t (&out)[32]) {
  float x[64];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint4 raw = *reinterpret_cast<const uint4*>(tile + rowo[q]);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[8 * q + 2 * e] = bf16_lo(w[e]);
      x[8 * q + 2 * e + 1] = bf16_hi(w[e]);
    }
  }
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = x[i];
#pragma unroll
  for (int i = 8; i < 64; ++i) mx[i & 7] = fmaxf(mx[i & 7], x[i]);
  float m = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
  xmax[h][t] = m;
  named_bar(1, 128);
  m = fmaxf(m, xmax[h ^ 1][t]);
  float inv = 1.0f;
  if (!elu1) {
    const float ml = m * kLog2e;
    float sp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      x[i] = ex2(fmaf(x[i], kLog2e, -ml));
      sp[i & 7] += x[i];
    }
    const float s = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
    xsum[h][t] = s;
    named_bar(1, 128);
    inv = 1.0f / (s + xsum[h ^ 1][t]);
  } else {
#pragma unroll
    for (int i = 0; i < 64; ++i) x[i] = x[i] > 0.0f ? x[i] + 1.0f : expf(x[i]);
    named_bar(1, 128);  // keeps the barrier sequence of both maps identical
  }
  const bool live = t < n;
#pragma unroll
  for (int i = 0; i < 32; ++i) out[i] = live ? pack_bf16(x[2 * i] * inv, x[2 * i + 1] * inv) : 0u;
}

// Column c of a block tile summed over all 64 rows, four interleaved partial
// sums (fixed order, so the result is deterministic).
__device__ __forceinline__ float sum_column(const unsigned char* tile, const uint32_t (&colo)[8]) {
  float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int t = 0; t < kBlock; ++t) p[t & 3] += elem_at(tile, colo, t);
  return (p[0] + p[1]) + (p[2] + p[3]);
}

__device__ __forceinline__ void store_half_row(unsigned char* tile, const uint32_t (&rowo)[8], const uint32_t (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<uint4*>(tile + rowo[q]) = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

}  // namespace

struct QStreamMaps {
  CUtensorMap q, phiq;
};
struct KvStreamMaps {
  CUtensorMap k, v, phik;
};

// ---------------------------------------------------------------------------
// Q side
// ---------------------------------------------------------------------------
struct QStreamArgs {
  const __nv_bfloat16* proj;  // SLA2 router proj_q [d][d], or null
  float* qbar;                // [BH][Nb][d]
  int* status;
  int N, Nb, cb;              // cb: blocks per chunk
  int want_phi, phi_elu1;
};

__global__ void __launch_bounds__(160, 3) q_stream_kernel(const __grid_constant__ QStreamMaps maps,
                                                          const QStreamArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[2 * kQStages];
  __shared__ int abort_sh;
  __shared__ __align__(16) float xbar[kRouterBatch][SD];  // read as float4 rows
  __shared__ float xmax[2][64], xsum[2][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int jb0 = chunk * a.cb;
  const int nblk = min(a.Nb, jb0 + a.cb) - jb0;
  volatile int* abort_flag = &abort_sh;
  auto bar = [&](int b) { return smem_u32(&bars[b]); };
  auto wait = [&](int b, uint32_t parity) { return mbar_wait(bar(b), parity, abort_flag, a.status); };
  int no_abort = 0;
  auto wait_drain = [&](int b, uint32_t parity) {
    return mbar_wait(bar(b), parity, reinterpret_cast<volatile int*>(&no_abort), a.status);
  };
  const uint32_t sb = smem_u32(smem);
  constexpr int kFull = 0, kEmpty = kQStages;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(bar(kFull + s), 1);
      mbar_init(bar(kEmpty + s), 1);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == 4) {
    // producer: block j into stage j % kQStages once its previous block is done
    bool stop = false;
    int issued = 0;
    if (lane == 0) prefetch_tmap(&maps.q);
    for (int j = 0; j < nblk; ++j) {
      const int s = j % kQStages;
      const bool ok = wait(kEmpty + s, ((j / kQStages) & 1) ^ 1) && *abort_flag == 0;
      stop = !__all_sync(0xffffffffu, ok);
      if (stop) break;
      if (lane == 0) {
        mbar_expect_tx(bar(kFull + s), kTileBytes);
        tma_load_3d(sb + s * kTileBytes, &maps.q, bar(kFull + s), 0, (jb0 + j) * kBlock, bh);
        tma_load_3d(sb + s * kTileBytes + kSub, &maps.q, bar(kFull + s), 64, (jb0 + j) * kBlock, bh);
      }
      issued = j + 1;
      __syncwarp();
    }
    // the last copy of every stage has landed before the CTA exits
    if (lane == 0)
      for (int j = issued > kQStages ? issued - kQStages : 0; j < issued; ++j)
        wait_drain(kFull + j % kQStages, (j / kQStages) & 1);
    __syncwarp();
  } else {
    // compute warps: thread t owns column t (pooling) and half t / 64 of row
    // t % 64 (phi)
    const int tid = threadIdx.x;
    const int r = tid & 63, h = tid >> 6;
    uint32_t colo[8], rowo[8];
    column_offsets(tid, colo);
#pragma unroll
    for (int q = 0; q < 8; ++q) rowo[q] = chunk_off(h, r, q);
    for (int j = 0; j < nblk; ++j) {
      const int s = j % kQStages;
      const int jb = jb0 + j;
      const int n = min(kBlock, a.N - jb * kBlock);
      wait(kFull + s, (j / kQStages) & 1);
      unsigned char* tile = smem + s * kTileBytes;
      const float pooled = pool_column(tile, colo, tid, n);
      if (a.proj) xbar[j % kRouterBatch][tid] = pooled;
      else a.qbar[(size_t(bh) * a.Nb + jb) * SD + tid] = pooled;
      if (a.want_phi) {
        // phi(Q) rows over the tile they come from (every read of the tile
        // happened before the barriers inside), then out by TMA store; the
        // stage is released once the store has read it
        uint32_t phv[32];
        phi_row_half(tile, rowo, r, h, n, a.phi_elu1 != 0, xmax, xsum, phv);
        store_half_row(tile, rowo, phv);
        fence_async_smem();
        named_bar(1, 128);
        if (tid == 0) {
          tma_store_3d(&maps.phiq, smem_u32(tile), 0, jb * kBlock, bh);
          tma_store_3d(&maps.phiq, smem_u32(tile) + kSub, 64, jb * kBlock, bh);
          bulk_commit();
          // the store of block j - 1 has read its stage: release that one
          // (block j's is released one block later, so this block's store
          // overlaps the next block's work)
          if (j > 0) {
            bulk_wait_read<1>();
            mbar_arrive(bar(kEmpty + (j - 1) % kQStages));
          }
          if (j == nblk - 1) {
            bulk_wait_read<0>();
            mbar_arrive(bar(kEmpty + s));
          }
        }
      } else {
        named_bar(1, 128);
        if (tid == 0) mbar_arrive(bar(kEmpty + s));
      }
      // router over a full batch (or the chunk's last blocks); the barriers
      // above made the batch's pooled rows visible, the one below keeps the
      // next batch from overwriting them while they are read
      if (a.proj && (j % kRouterBatch == kRouterBatch - 1 || j == nblk - 1)) {
        const int j0 = j - j % kRouterBatch;
        router_batch(xbar, j - j0 + 1, a.proj, tid, a.qbar + (size_t(bh) * a.Nb + jb0 + j0) * SD, SD);
        named_bar(1, 128);
      }
    }
    if (tid == 0) bulk_wait_all();
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// K / V side
// ---------------------------------------------------------------------------
struct KvStreamArgs {
  const __nv_bfloat16* proj;  // SLA2 router proj_k [d][d], or null
  float* kbar;                // [BH][Nb][d]
  float* zblk;                // [BH][Nb][d]
  float* hpart;               // [BH][nchunk][d][d]
  float* zpart;               // [BH][nchunk][d]
  int* status;
  int N, Nb, cb, nchunk;
  int phi_elu1;
};

enum KvBar { kvFull0 = 0, kvEmpty0 = kvFull0 + kKvStages, kvPhiFull0 = kvEmpty0 + kKvStages,
             kvDone = kvPhiFull0 + kKvStages, kvNumBars };

__global__ void __launch_bounds__(192, 2) kv_stream_kernel(const __grid_constant__ KvStreamMaps maps,
                                                           const KvStreamArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[kvNumBars];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ __align__(16) float xbar[kRouterBatch][SD];  // read as float4 rows
  __shared__ float xmax[2][64], xsum[2][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int jb0 = chunk * a.cb;
  const int nblk = min(a.Nb, jb0 + a.cb) - jb0;
  volatile int* abort_flag = &abort_sh;
  auto bar = [&](int b) { return smem_u32(&bars[b]); };
  auto wait = [&](int b, uint32_t parity) { return mbar_wait(bar(b), parity, abort_flag, a.status); };
  auto wait_w = [&](int b, uint32_t parity) {
    const bool ok = wait(b, parity);
    __syncwarp();
    return ok;
  };
  int no_abort = 0;
  auto wait_drain = [&](int b, uint32_t parity) {
    return mbar_wait(bar(b), parity, reinterpret_cast<volatile int*>(&no_abort), a.status);
  };
  const uint32_t sb = smem_u32(smem);
  // stage s: K tile (later phi(K), written over it) at s * 2 tiles, V tile right after it
  auto ktile = [&](int s) { return s * 2 * kTileBytes; };
  auto vtile = [&](int s) { return s * 2 * kTileBytes + kTileBytes; };

  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int s = 0; s < kKvStages; ++s) {
      mbar_init(bar(kvFull0 + s), 1);
      // the compute warps (phi read back, phi stored) and the product (phi, V read)
      mbar_init(bar(kvEmpty0 + s), 2);
      mbar_init(bar(kvPhiFull0 + s), 1);
    }
    mbar_init(bar(kvDone), 1);
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(smem_u32(&tmem_base_sh), 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tmem_base_sh;

  if (warp == 4) {
    // producer: K and V of block j into stage j % kKvStages
    bool stop = false;
    int issued = 0;
    if (lane == 0) {
      prefetch_tmap(&maps.k);
      prefetch_tmap(&maps.v);
    }
    for (int j = 0; j < nblk; ++j) {
      const int s = j % kKvStages;
      const bool ok = wait(kvEmpty0 + s, ((j / kKvStages) & 1) ^ 1) && *abort_flag == 0;
      stop = !__all_sync(0xffffffffu, ok);
      if (stop) break;
      if (lane == 0) {
        const int y = (jb0 + j) * kBlock;
        mbar_expect_tx(bar(kvFull0 + s), 2 * kTileBytes);
        tma_load_3d(sb + ktile(s), &maps.k, bar(kvFull0 + s), 0, y, bh);
        tma_load_3d(sb + ktile(s) + kSub, &maps.k, bar(kvFull0 + s), 64, y, bh);
        tma_load_3d(sb + vtile(s), &maps.v, bar(kvFull0 + s), 0, y, bh);
        tma_load_3d(sb + vtile(s) + kSub, &maps.v, bar(kvFull0 + s), 64, y, bh);
      }
      issued = j + 1;
      __syncwarp();
    }
    if (lane == 0)
      for (int j = issued > kKvStages ? issued - kKvStages : 0; j < issued; ++j)
        wait_drain(kvFull0 + j % kKvStages, (j / kKvStages) & 1);
    __syncwarp();
  } else if (warp == 5) {
    // H += phi(K_j)^T V_j: M = N = d, K = 64 tokens, both operands MN-major
    // (tokens are the rows of both tiles); 4 instructions of K = 16
    constexpr uint32_t idH = idesc_bf16(SD, SD, 1, 1);
    for (int j = 0; j < nblk; ++j) {
      const int s = j % kKvStages;
      wait_w(kvFull0 + s, (j / kKvStages) & 1);     // V landed
      wait_w(kvPhiFull0 + s, (j / kKvStages) & 1);  // phi(K) written over K
      tc_fence_after();
      const uint32_t pa = sb + ktile(s), vb = sb + vtile(s);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16(tb, sdesc(pa + k * 2048, kSub, 1024), sdesc(vb + k * 2048, kSub, 1024), idH,
                 (j > 0 || k > 0) ? 1u : 0u);
      mma_commit(bar(kvEmpty0 + s));
    }
    mma_commit(bar(kvDone));
    wait_drain(kvDone, 0);
    __syncwarp();
  } else {
    const int tid = threadIdx.x;
    const int r = tid & 63, h = tid >> 6;
    const bool elu1 = a.phi_elu1 != 0;
    uint32_t colo[8], rowo[8];
    column_offsets(tid, colo);
#pragma unroll
    for (int q = 0; q < 8; ++q) rowo[q] = chunk_off(h, r, q);
    float zacc = 0.0f;
    for (int j = 0; j < nblk; ++j) {
      const int s = j % kKvStages;
      const int jb = jb0 + j;
      const int n = min(kBlock, a.N - jb * kBlock);
      wait(kvFull0 + s, (j / kKvStages) & 1);
      unsigned char* kt = smem + ktile(s);
      const float pooled = pool_column(kt, colo, tid, n);
      if (a.proj) xbar[j % kRouterBatch][tid] = pooled;
      else a.kbar[(size_t(bh) * a.Nb + jb) * SD + tid] = pooled;
      uint32_t phv[32];
      phi_row_half(kt, rowo, r, h, n, elu1, xmax, xsum, phv);
      // every read of K happened before the barriers inside phi_row_half:
      // phi(K) goes over it, in the same layout (the product's A operand)
      store_half_row(kt, rowo, phv);
      fence_async_smem();
      named_bar(1, 128);
      if (tid == 0) {
        mbar_arrive(bar(kvPhiFull0 + s));
        tma_store_3d(&maps.phik, smem_u32(kt), 0, jb * kBlock, bh);
        tma_store_3d(&maps.phik, smem_u32(kt) + kSub, 64, jb * kBlock, bh);
        bulk_commit();
      }
      // z_j: column tid of the bf16 phi tile (rows past N hold zero)
      const float z = sum_column(kt, colo);
      a.zblk[(size_t(bh) * a.Nb + jb) * SD + tid] = z;
      zacc += z;
      if (a.proj && (j % kRouterBatch == kRouterBatch - 1 || j == nblk - 1)) {
        const int j0 = j - j % kRouterBatch;
        router_batch(xbar, j - j0 + 1, a.proj, tid, a.kbar + (size_t(bh) * a.Nb + jb0 + j0) * SD, SD);
      }
      // all z reads of the tile are done; the store has read it: release the stage
      named_bar(1, 128);
      if (tid == 0) {
        bulk_wait_read<0>();
        mbar_arrive(bar(kvEmpty0 + s));
      }
    }
    // the chunk's partial H (TMEM lane = row of H) and Z
    wait(kvDone, 0);
    __syncwarp();
    tc_fence_after();
    float* hp = a.hpart + (size_t(bh) * a.nchunk + chunk) * SD * SD + size_t(tid) * SD;
    const uint32_t tq = tb + (uint32_t(32 * warp) << 16);
#pragma unroll 1
    for (int c = 0; c < SD / 32; ++c) {
      float v[32];
      tmem_ld32(tq + c * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float4*>(hp + c * 32 + 4 * q) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
    a.zpart[(size_t(bh) * a.nchunk + chunk) * SD + tid] = zacc;
    if (tid == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tb, 128);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
int stream_smem_q() { return kQStages * kTileBytes + 1024; }
int stream_smem_kv() { return kKvStages * 2 * kTileBytes + 1024; }

cudaError_t launch_q_stream(const Layout& L, const __nv_bfloat16* Q, const __nv_bfloat16* proj_q, float* qbar,
                            __nv_bfloat16* phiq, int phi_elu1, int* status, cudaStream_t s) {
  QStreamMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (!map_rows(&maps.q, Q, SD, L.N, L.Npad, L.BH)) return cudaErrorInvalidValue;
  if (phiq && !map_rows(&maps.phiq, phiq, SD, L.N, L.Npad, L.BH)) return cudaErrorInvalidValue;
  // the Q pass keeps no partial sums, so its chunks are sized on their own:
  // about three CTAs per SM (its shared memory allows three)
  const int per_head = std::max(1, std::min(L.Nb, 3 * (kStreamCtas / 2) / std::max(1, L.BH)));
  const int cb = (L.Nb + per_head - 1) / per_head;
  const int nchunk = (L.Nb + cb - 1) / cb;
  QStreamArgs a{proj_q, qbar, status, L.N, L.Nb, cb, phiq != nullptr ? 1 : 0, phi_elu1};
  const int bytes = stream_smem_q();
  cudaError_t e = cudaFuncSetAttribute(q_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  q_stream_kernel<<<dim3(nchunk, L.BH), 160, bytes, s>>>(maps, a);
  return cudaGetLastError();
}

cudaError_t launch_kv_stream(const Layout& L, const __nv_bfloat16* K, const __nv_bfloat16* V,
                             const __nv_bfloat16* proj_k, float* kbar, __nv_bfloat16* phik, float* zblk,
                             float* hpart, float* zpart, int phi_elu1, int* status, cudaStream_t s) {
  KvStreamMaps maps;
  memset(&maps, 0, sizeof(maps));
  // phi(K) rows past N are stored as zeros (the attention kernel reads whole blocks)
  if (!map_rows(&maps.k, K, SD, L.N, L.Npad, L.BH) || !map_rows(&maps.v, V, SD, L.N, L.Npad, L.BH) ||
      !map_rows(&maps.phik, phik, SD, L.Npad, L.Npad, L.BH))
    return cudaErrorInvalidValue;
  KvStreamArgs a{proj_k, kbar, zblk, hpart, zpart, status, L.N, L.Nb, L.stream_cb, L.nchunk, phi_elu1};
  const int bytes = stream_smem_kv();
  cudaError_t e = cudaFuncSetAttribute(kv_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  kv_stream_kernel<<<dim3(L.nchunk, L.BH), 192, bytes, s>>>(maps, a);
  return cudaGetLastError();
}

}  // namespace sla
