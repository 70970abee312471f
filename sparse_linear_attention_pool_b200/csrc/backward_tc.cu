// The sparse (critical-block) loops of the backward pass on the 5th-generation
// tensor cores (tcgen05 / TMEM / TMA), d = 128, bf16. Source: SLA walkthrough
// (intelliparadigm.com), section 2.3: the sparse path takes the FlashAttention
// backward on the Mc = 1 blocks; the linear path's gradients are added by the
// mma.sync kernels of backward_kernels.cu, which also take these partials.
//
// dK / dV (bwd_kv_tc_kernel): one CTA per pair of key blocks (j_A = 2c,
// j_B = 2c + 1); the 128 key rows sit in TMEM lanes 0-127 (j_A's then j_B's).
// The CTA walks the union of the two blocks' column lists (the query blocks i
// with j_A or j_B critical), in ascending i; every role merges the two lists
// with its own two pointers. Per query block i:
//   S^T  = [K_jA; K_jB] Q_i^T   (M = 128, N = 64, K = d)   -> TMEM cols 0-63
//   dP^T = [V_jA; V_jB] dO_i^T  (M = 128, N = 64, K = d)   -> TMEM cols 64-127
//   P^T  = exp(scale S^T - lse_i), 0 in the rows whose key block does not have
//          i critical (and past N); dS^T = P^T (asc dP^T - D_i)    (softmax warps)
//   dV  += P^T dO_i  (M = 128, N = d, K = 64)                 -> TMEM cols 128-255
//   dK  += dS^T Q_i  (M = 128, N = d, K = 64)                 -> TMEM cols 256-383
// Q_i and dO_i are one SW128 tile each: K-major as the B operand of S^T / dP^T,
// MN-major as the B operand of dK / dV. The sparse partials leave as fp32
// (dK scaled by the softmax scale, dV by asc = alpha_h for SLA2, 1 for SLA).
//
// dQ (bwd_q_tc_kernel): the mirror, one CTA per pair of query blocks over the
// union of their critical lists, dQ += dS K_j accumulated in TMEM.
//
// Warp roles as in the forward's attention kernel: warp 4 issues the copies,
// warp 5 the MMAs (and owns TMEM), warps 0-3 turn S / dP into P / dS. Every
// wait is bounded; the producer waits for its last copies before exiting.
#include <string.h>

#include "tc_util.cuh"

namespace sla {

using namespace tc;

namespace {

constexpr int kSub64 = 64 * 128;    // 8 KB: 64 rows x 128 B (one 64-column SW128 sub-tile of a 64-row tile)
constexpr int kSub128 = 128 * 128;  // 16 KB: 128 rows x 128 B
constexpr int kTile64 = 2 * kSub64; // 16 KB: a 64 x 128 bf16 tile
constexpr int oK = 0;                       // K pair: 2 sub-tiles of 128 rows (j_A rows, then j_B rows at +kSub64)
constexpr int oV = oK + 2 * kSub128;        // V pair
constexpr int oQ = oV + 2 * kSub128;        // Q ring: 2 stages
constexpr int oO = oQ + 2 * kTile64;        // dO ring: 2 stages
constexpr int oP = oO + 2 * kTile64;        // P^T: [128 rows][64 queries] bf16, SW128
constexpr int oS = oP + kSub128;            // dS^T: same
constexpr int oL = oS + kSub128;            // per stage: lse (64 floats), D (64 floats)
constexpr int kBytes = oL + 2 * 512;        // 161 KB
constexpr int kSmem = kBytes + 1024;        // + alignment slack
constexpr int cS = 0, cP = 64, cV = 128, cK = 256;
constexpr uint32_t kCols = 512;

enum { bKV = 0, bQFull0, bQFull1, bQEmpty0, bQEmpty1, bSFull, bSFree, bPFull, bPDone, bDone, kBars };

struct KvTcMaps {
  CUtensorMap q, k, v, o;
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

struct Union {  // ascending merge of two ascending lists
  const int *la, *lb;
  int na, nb, pa = 0, pb = 0;
  __device__ bool next(int& i, bool& inA, bool& inB) {
    if (pa >= na && pb >= nb) return false;
    const int ia = pa < na ? la[pa] : 0x7fffffff, ib = pb < nb ? lb[pb] : 0x7fffffff;
    i = ia < ib ? ia : ib;
    inA = ia == i;
    inB = ib == i;
    pa += inA;
    pb += inB;
    return true;
  }
};

}  // namespace

__global__ void __launch_bounds__(192, 1) bwd_kv_tc_kernel(const __grid_constant__ KvTcMaps maps, const KvTcArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[kBars];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, h = bh % a.H;
  const int jA = 2 * blockIdx.x, jB = jA + 1;
  const bool validB = jB < a.Nb;
  const int nA = a.cntC[size_t(bh) * a.Nb + jA], nB = validB ? a.cntC[size_t(bh) * a.Nb + jB] : 0;
  const int* lA = a.colC + (size_t(bh) * a.Nb + jA) * a.Nb;
  const int* lB = validB ? a.colC + (size_t(bh) * a.Nb + jB) * a.Nb : lA;
  volatile int* abort_flag = &abort_sh;
  auto bar = [&](int b) { return smem_u32(&bars[b]); };
  auto wait = [&](int b, uint32_t parity) { return mbar_wait(bar(b), parity, abort_flag, a.status); };
  auto wait_w = [&](int b, uint32_t parity) {
    const bool ok = wait(b, parity);
    __syncwarp();
    return ok;
  };
  const uint32_t sb = smem_u32(smem);
  // bounded waits that ignore the abort flag: in-flight copies / MMAs must land before exit
  int no_abort = 0;
  auto wait_drain = [&](int b, uint32_t parity) {
    return mbar_wait(bar(b), parity, reinterpret_cast<volatile int*>(&no_abort), a.status);
  };

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(bar(bKV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(bQFull0 + s), 1);
      mbar_init(bar(bQEmpty0 + s), 1);
    }
    mbar_init(bar(bSFull), 1);
    mbar_init(bar(bSFree), 128);
    mbar_init(bar(bPFull), 128);
    mbar_init(bar(bPDone), 1);
    mbar_init(bar(bDone), 1);
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(smem_u32(&tmem_base_sh), kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tmem_base_sh;

  if (warp == 4) {
    // producer: K and V pairs once, then per union step the Q and dO tiles of i
    // and its lse / D rows (two 256-byte bulk copies) on the stage's barrier
    if (lane == 0) {
      mbar_expect_tx(bar(bKV), 4 * kSub128);
      for (int s = 0; s < 2; ++s) {
        tma_load_3d(sb + oK + s * kSub128, &maps.k, bar(bKV), s * 64, jA * 64, bh);
        tma_load_3d(sb + oK + s * kSub128 + kSub64, &maps.k, bar(bKV), s * 64, jB * 64, bh);
        tma_load_3d(sb + oV + s * kSub128, &maps.v, bar(bKV), s * 64, jA * 64, bh);
        tma_load_3d(sb + oV + s * kSub128 + kSub64, &maps.v, bar(bKV), s * 64, jB * 64, bh);
      }
      Union u{lA, lB, nA, nB};
      int i, issued = 0;
      bool inA, inB;
      for (int t = 0; u.next(i, inA, inB); ++t) {
        const int st = t & 1;
        if (!wait(bQEmpty0 + st, ((t >> 1) & 1) ^ 1)) break;
        issued = t + 1;
        const uint32_t fb = bar(bQFull0 + st);
        mbar_expect_tx(fb, 2 * kTile64 + 512);
        for (int s = 0; s < 2; ++s) {
          tma_load_3d(sb + oQ + st * kTile64 + s * kSub64, &maps.q, fb, s * 64, i * 64, bh);
          tma_load_3d(sb + oO + st * kTile64 + s * kSub64, &maps.o, fb, s * 64, i * 64, bh);
        }
        const size_t row0 = size_t(bh) * a.Npad + size_t(i) * 64;
        bulk_load(sb + oL + st * 512, a.lse + row0, 256, fb);
        bulk_load(sb + oL + st * 512 + 256, a.Drow + row0, 256, fb);
      }
      // the last copies have landed before the CTA can exit (an aborted run included)
      wait_drain(bKV, 0);
      for (int tt = issued > 2 ? issued - 2 : 0; tt < issued; ++tt) wait_drain(bQFull0 + (tt & 1), (tt >> 1) & 1);
    }
    __syncwarp();
  } else if (warp == 5) {
    // MMA issuer: S^T(t), dP^T(t), then dV / dK of step t - 1
    constexpr uint32_t idS = idesc_bf16(128, 64, 0, 0);
    constexpr uint32_t idD = idesc_bf16(128, 128, 0, 1);
    wait_w(bKV, 0);
    tc_fence_after();
    auto issue_dvdk = [&](int tp) {
      const int st = tp & 1;
      wait_w(bPFull, tp & 1);
      tc_fence_after();
      const uint32_t sq = sb + oQ + st * kTile64, so = sb + oO + st * kTile64;
#pragma unroll
      for (int k = 0; k < 4; ++k) {  // K = 64 queries, 16 per instruction
        const uint32_t acc = (tp > 0 || k > 0) ? 1u : 0u;
        mma_bf16(tb + cV, sdesc(sb + oP + k * 32, 16, 1024), sdesc(so + k * 2048, kSub64, 1024), idD, acc);
        mma_bf16(tb + cK, sdesc(sb + oS + k * 32, 16, 1024), sdesc(sq + k * 2048, kSub64, 1024), idD, acc);
      }
      mma_commit(bar(bQEmpty0 + st));
      mma_commit(bar(bPDone));
    };
    Union u{lA, lB, nA, nB};
    int i, t = 0;
    bool inA, inB;
    for (; u.next(i, inA, inB); ++t) {
      const int st = t & 1;
      wait_w(bQFull0 + st, (t >> 1) & 1);
      wait_w(bSFree, (t & 1) ^ 1);
      tc_fence_after();
      const uint32_t sq = sb + oQ + st * kTile64, so = sb + oO + st * kTile64;
#pragma unroll
      for (int k = 0; k < 8; ++k) {  // K = d = 128, 16 per instruction
        const uint32_t offA = (k >> 2) * kSub128 + (k & 3) * 32, offB = (k >> 2) * kSub64 + (k & 3) * 32;
        mma_bf16(tb + cS, sdesc(sb + oK + offA, 16, 1024), sdesc(sq + offB, 16, 1024), idS, k > 0);
        mma_bf16(tb + cP, sdesc(sb + oV + offA, 16, 1024), sdesc(so + offB, 16, 1024), idS, k > 0);
      }
      mma_commit(bar(bSFull));
      if (t > 0) issue_dvdk(t - 1);
    }
    if (t > 0) issue_dvdk(t - 1);
    mma_commit(bar(bDone));
    wait_drain(bDone, 0);  // every product has completed before TMEM is released
    __syncwarp();
  } else {
    // softmax warps: key row r = TMEM lane
    const int r = threadIdx.x;
    const uint32_t tq = tb + (uint32_t(32 * warp) << 16);
    const int nvA = min(64, a.N - jA * 64), nvB = validB ? min(64, a.N - jB * 64) : 0;
    const bool vrow = r < 64 ? r < nvA : (r - 64) < nvB;
    const float asc = a.alpha ? a.alpha[h] : 1.0f;
    Union u{lA, lB, nA, nB};
    int i, t = 0;
    bool inA, inB;
    for (; u.next(i, inA, inB); ++t) {
      const int st = t & 1;
      wait_w(bSFull, t & 1);
      tc_fence_after();
      float s[64], dp[64];
      {
        float x[32];
        tmem_ld32(tq + cS, x);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) s[c] = x[c];
        tmem_ld32(tq + cS + 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) s[32 + c] = x[c];
        tmem_ld32(tq + cP, x);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) dp[c] = x[c];
        tmem_ld32(tq + cP + 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) dp[32 + c] = x[c];
      }
      tc_fence_before();
      mbar_arrive(bar(bSFree));
      // this step's lse / D rows arrived with the Q tile (stage barrier already complete)
      wait(bQFull0 + st, (t >> 1) & 1);
      const float* lrow = reinterpret_cast<const float*>(smem + oL + st * 512);
      const float* drow = lrow + 64;
      const int nvi = min(64, a.N - i * 64);
      const bool live = vrow && (r < 64 ? inA : inB);
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const bool on = live && c < nvi;  // lse / D past N are not written: select, never multiply by 0
        const float p = on ? ex2(fmaf(s[c], a.scale_log2, -lrow[c] * kLog2e)) : 0.0f;
        s[c] = p;
        dp[c] = on ? p * (asc * dp[c] - drow[c]) : 0.0f;
      }
      if (t >= 1) wait(bPDone, (t - 1) & 1);  // P^T / dS^T of step t - 1 have been read
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        *reinterpret_cast<uint4*>(smem + oP + sw128_chunk(r, c8)) =
            make_uint4(pack_bf16(s[8 * c8], s[8 * c8 + 1]), pack_bf16(s[8 * c8 + 2], s[8 * c8 + 3]),
                       pack_bf16(s[8 * c8 + 4], s[8 * c8 + 5]), pack_bf16(s[8 * c8 + 6], s[8 * c8 + 7]));
        *reinterpret_cast<uint4*>(smem + oS + sw128_chunk(r, c8)) =
            make_uint4(pack_bf16(dp[8 * c8], dp[8 * c8 + 1]), pack_bf16(dp[8 * c8 + 2], dp[8 * c8 + 3]),
                       pack_bf16(dp[8 * c8 + 4], dp[8 * c8 + 5]), pack_bf16(dp[8 * c8 + 6], dp[8 * c8 + 7]));
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar(bPFull));
    }
    // the sparse partials: dV (x asc), dK (x scale), fp32, valid key rows only
    wait_w(bDone, 0);
    tc_fence_after();
    const int krow = (r < 64 ? jA * 64 + r : jB * 64 + (r - 64));
    float* dv = a.dVs + (size_t(bh) * a.Npad + krow) * 128;
    float* dk = a.dKs + (size_t(bh) * a.Npad + krow) * 128;
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
      float x[32], y[32];
      if (t > 0) {
        tmem_ld32(tq + cV + ch * 32, x);
        tmem_ld32(tq + cK + ch * 32, y);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c] = y[c] = 0.0f;
      }
      if (vrow) {
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          *reinterpret_cast<float4*>(dv + ch * 32 + c) = make_float4(x[c] * asc, x[c + 1] * asc, x[c + 2] * asc, x[c + 3] * asc);
          *reinterpret_cast<float4*>(dk + ch * 32 + c) =
              make_float4(y[c] * a.scale, y[c + 1] * a.scale, y[c + 2] * a.scale, y[c + 3] * a.scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tb, kCols);
  }
}

// dQ mirror: one CTA per pair of query blocks (i_A, i_B), rows = 128 queries in
// TMEM lanes; it walks the union of the two critical lists (the key blocks j
// critical for i_A or i_B). Per key block j: S = [Q_A; Q_B] K_j^T and
// dP = [dO_A; dO_B] V_j^T (M = 128, N = 64), dS = P (asc dP - D_r) with P = 0
// in the row half whose block does not have j critical and past N, then
// dQ += dS K_j (M = 128, N = d, K = 64 keys; K_j MN-major). fp32 partial,
// scaled by the softmax scale.
__global__ void __launch_bounds__(192, 1) bwd_q_tc_kernel(const __grid_constant__ KvTcMaps maps, const QTcArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[kBars];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, h = bh % a.H;
  const int iA = 2 * blockIdx.x, iB = iA + 1;
  const bool validB = iB < a.Nb;
  const int* lA = a.crit + (size_t(bh) * a.Nb + iA) * a.kc;
  const int* lB = validB ? a.crit + (size_t(bh) * a.Nb + iB) * a.kc : lA;
  const int nA = a.kc, nB = validB ? a.kc : 0;
  volatile int* abort_flag = &abort_sh;
  auto bar = [&](int b) { return smem_u32(&bars[b]); };
  auto wait = [&](int b, uint32_t parity) { return mbar_wait(bar(b), parity, abort_flag, a.status); };
  auto wait_w = [&](int b, uint32_t parity) {
    const bool ok = wait(b, parity);
    __syncwarp();
    return ok;
  };
  const uint32_t sb = smem_u32(smem);
  int no_abort = 0;
  auto wait_drain = [&](int b, uint32_t parity) {
    return mbar_wait(bar(b), parity, reinterpret_cast<volatile int*>(&no_abort), a.status);
  };
  // smem: Q pair (oK slot), dO pair (oV slot), K_j / V_j ring (oQ / oO), dS (oS)
  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(bar(bKV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(bQFull0 + s), 1);
      mbar_init(bar(bQEmpty0 + s), 1);
    }
    mbar_init(bar(bSFull), 1);
    mbar_init(bar(bSFree), 128);
    mbar_init(bar(bPFull), 128);
    mbar_init(bar(bPDone), 1);
    mbar_init(bar(bDone), 1);
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(smem_u32(&tmem_base_sh), kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tmem_base_sh;

  if (warp == 4) {
    if (lane == 0) {
      mbar_expect_tx(bar(bKV), 4 * kSub128);
      for (int s = 0; s < 2; ++s) {
        tma_load_3d(sb + oK + s * kSub128, &maps.q, bar(bKV), s * 64, iA * 64, bh);
        tma_load_3d(sb + oK + s * kSub128 + kSub64, &maps.q, bar(bKV), s * 64, iB * 64, bh);
        tma_load_3d(sb + oV + s * kSub128, &maps.o, bar(bKV), s * 64, iA * 64, bh);
        tma_load_3d(sb + oV + s * kSub128 + kSub64, &maps.o, bar(bKV), s * 64, iB * 64, bh);
      }
      Union u{lA, lB, nA, nB};
      int j, issued = 0;
      bool inA, inB;
      for (int t = 0; u.next(j, inA, inB); ++t) {
        const int st = t & 1;
        if (!wait(bQEmpty0 + st, ((t >> 1) & 1) ^ 1)) break;
        issued = t + 1;
        const uint32_t fb = bar(bQFull0 + st);
        mbar_expect_tx(fb, 2 * kTile64);
        for (int s = 0; s < 2; ++s) {
          tma_load_3d(sb + oQ + st * kTile64 + s * kSub64, &maps.k, fb, s * 64, j * 64, bh);
          tma_load_3d(sb + oO + st * kTile64 + s * kSub64, &maps.v, fb, s * 64, j * 64, bh);
        }
      }
      wait_drain(bKV, 0);
      for (int tt = issued > 2 ? issued - 2 : 0; tt < issued; ++tt) wait_drain(bQFull0 + (tt & 1), (tt >> 1) & 1);
    }
    __syncwarp();
  } else if (warp == 5) {
    constexpr uint32_t idS = idesc_bf16(128, 64, 0, 0);
    constexpr uint32_t idD = idesc_bf16(128, 128, 0, 1);
    wait_w(bKV, 0);
    tc_fence_after();
    auto issue_dq = [&](int tp) {
      const int st = tp & 1;
      wait_w(bPFull, tp & 1);
      tc_fence_after();
      const uint32_t sk = sb + oQ + st * kTile64;
#pragma unroll
      for (int k = 0; k < 4; ++k) {  // K = 64 keys
        const uint32_t acc = (tp > 0 || k > 0) ? 1u : 0u;
        mma_bf16(tb + cV, sdesc(sb + oS + k * 32, 16, 1024), sdesc(sk + k * 2048, kSub64, 1024), idD, acc);
      }
      mma_commit(bar(bQEmpty0 + st));
      mma_commit(bar(bPDone));
    };
    Union u{lA, lB, nA, nB};
    int j, t = 0;
    bool inA, inB;
    for (; u.next(j, inA, inB); ++t) {
      const int st = t & 1;
      wait_w(bQFull0 + st, (t >> 1) & 1);
      wait_w(bSFree, (t & 1) ^ 1);
      tc_fence_after();
      const uint32_t sk = sb + oQ + st * kTile64, sv = sb + oO + st * kTile64;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t offA = (k >> 2) * kSub128 + (k & 3) * 32, offB = (k >> 2) * kSub64 + (k & 3) * 32;
        mma_bf16(tb + cS, sdesc(sb + oK + offA, 16, 1024), sdesc(sk + offB, 16, 1024), idS, k > 0);
        mma_bf16(tb + cP, sdesc(sb + oV + offA, 16, 1024), sdesc(sv + offB, 16, 1024), idS, k > 0);
      }
      mma_commit(bar(bSFull));
      if (t > 0) issue_dq(t - 1);
    }
    if (t > 0) issue_dq(t - 1);
    mma_commit(bar(bDone));
    wait_drain(bDone, 0);
    __syncwarp();
  } else {
    const int r = threadIdx.x;
    const uint32_t tq = tb + (uint32_t(32 * warp) << 16);
    const int nvA = min(64, a.N - iA * 64), nvB = validB ? min(64, a.N - iB * 64) : 0;
    const bool vrow = r < 64 ? r < nvA : (r - 64) < nvB;
    const int qrow = r < 64 ? iA * 64 + r : iB * 64 + (r - 64);
    const size_t grow = size_t(bh) * a.Npad + qrow;
    const float asc = a.alpha ? a.alpha[h] : 1.0f;
    const float lse2 = vrow ? a.lse[grow] * kLog2e : 0.0f;
    const float Dr = vrow ? a.Drow[grow] : 0.0f;
    Union u{lA, lB, nA, nB};
    int j, t = 0;
    bool inA, inB;
    for (; u.next(j, inA, inB); ++t) {
      wait_w(bSFull, t & 1);
      tc_fence_after();
      float s[64], dp[64];
      {
        float x[32];
        tmem_ld32(tq + cS, x);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) s[c] = x[c];
        tmem_ld32(tq + cS + 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) s[32 + c] = x[c];
        tmem_ld32(tq + cP, x);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) dp[c] = x[c];
        tmem_ld32(tq + cP + 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) dp[32 + c] = x[c];
      }
      tc_fence_before();
      mbar_arrive(bar(bSFree));
      const int nvj = min(64, a.N - j * 64);
      const bool live = vrow && (r < 64 ? inA : inB);
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const bool on = live && c < nvj;
        const float p = on ? ex2(fmaf(s[c], a.scale_log2, -lse2)) : 0.0f;
        dp[c] = on ? p * (asc * dp[c] - Dr) : 0.0f;
      }
      if (t >= 1) wait(bPDone, (t - 1) & 1);
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8)
        *reinterpret_cast<uint4*>(smem + oS + sw128_chunk(r, c8)) =
            make_uint4(pack_bf16(dp[8 * c8], dp[8 * c8 + 1]), pack_bf16(dp[8 * c8 + 2], dp[8 * c8 + 3]),
                       pack_bf16(dp[8 * c8 + 4], dp[8 * c8 + 5]), pack_bf16(dp[8 * c8 + 6], dp[8 * c8 + 7]));
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar(bPFull));
    }
    wait_w(bDone, 0);
    tc_fence_after();
    float* dq = a.dQs + grow * 128;
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
      float x[32];
      if (t > 0) {
        tmem_ld32(tq + cV + ch * 32, x);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c] = 0.0f;
      }
      if (vrow) {
#pragma unroll
        for (int c = 0; c < 32; c += 4)
          *reinterpret_cast<float4*>(dq + ch * 32 + c) =
              make_float4(x[c] * a.scale, x[c + 1] * a.scale, x[c + 2] * a.scale, x[c + 3] * a.scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tb, kCols);
  }
}

namespace {
typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeFn enc_fn() {
  static EncodeFn fn = nullptr;
  if (fn == nullptr) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  }
  return fn;
}
// [BH][Npad][128] bf16 as 3D (128, rows, BH), 64 x 64 SW128 boxes; rows >= N read as zero
bool map128(CUtensorMap* m, const void* base, int N, int Npad, int BH) {
  EncodeFn enc = enc_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, cuuint64_t(N), cuuint64_t(BH)};
  cuuint64_t strides[2] = {256, cuuint64_t(Npad) * 256};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

cudaError_t launch_bwd_q_tc(const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                            const __nv_bfloat16* dO, const QTcArgs& a, int BH, cudaStream_t s) {
  KvTcMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (!map128(&maps.q, Q, a.N, a.Npad, BH) || !map128(&maps.k, K, a.N, a.Npad, BH) ||
      !map128(&maps.v, V, a.N, a.Npad, BH) || !map128(&maps.o, dO, a.N, a.Npad, BH))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(bwd_q_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  bwd_q_tc_kernel<<<dim3((a.Nb + 1) / 2, BH), 192, kSmem, s>>>(maps, a);
  return cudaGetLastError();
}

cudaError_t launch_bwd_kv_tc(const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                             const __nv_bfloat16* dO, const KvTcArgs& a, int BH, cudaStream_t s) {
  KvTcMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (!map128(&maps.q, Q, a.N, a.Npad, BH) || !map128(&maps.k, K, a.N, a.Npad, BH) ||
      !map128(&maps.v, V, a.N, a.Npad, BH) || !map128(&maps.o, dO, a.N, a.Npad, BH))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(bwd_kv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  bwd_kv_tc_kernel<<<dim3((a.Nb + 1) / 2, BH), 192, kSmem, s>>>(maps, a);
  return cudaGetLastError();
}

}  // namespace sla
