// Hybrid compute and fusion on the 5th-generation tensor cores (tcgen05).
//
// One CTA handles two adjacent 64-row query blocks A and B of one head. Per
// query block i the method computes ([SLA-sum] = SLA structured summary,
// aipaper.cc, section 4; [SLA-walk] = SLA walkthrough, intelliparadigm.com):
//   O^s_i = softmax over the keys of the critical blocks of row i, scale
//           1/sqrt(d), by online softmax ([SLA-sum] step 3; [SLA-walk] 2.2);
//   O^l_i = phi(Q_i) H_i / phi(Q_i) Z_i, H_i and Z_i summed over the marginal
//           blocks ([SLA-sum] formula 3), formed here as
//           H_i = H_tot - G_i, G_i = sum_{j in E_i} phi(K_j)^T V_j and
//           Z_i = Z_tot - sum_{j in E_i} z_j, E_i = critical and negligible blocks;
//   SLA:  O = O^s + O^l W ([SLA-sum] formula 4);
//   SLA2: O = alpha_h O^s + (1 - alpha_h) O^l (SLA2 article, mcffsbgs.com,
//         mixing-formula paragraph).
// Dense mode (the baseline): every key block critical, O = O^s; both query
// blocks then read the same K/V tile at every step, which is loaded once.
//
// Warp roles (192 threads):
//   warps 0-3  softmax / epilogue: one thread per row of the pair (block A's
//              64 rows in TMEM lanes 0-63, block B's in lanes 64-127);
//   warp 4     TMA producer: Q tiles, then per step the K and V tiles of both
//              blocks (phase 1; bf16 at d = 128 also phi(K) into the K slot
//              once S has read it), then the phi(K) / V tiles of the remaining
//              excluded blocks (phase 2), then phi(Q) over the Q tiles, then W;
//   warp 5     MMA issuer and TMEM owner: the converged warp walks the loop,
//              one elected lane issues each MMA and commit.
// K tiles and V tiles travel in separate rings: a K slot is released as soon
// as the S products that read it complete, a V slot after its PV product.
// Phase 1 per step t, over the 128-row pair [Q_A; Q_B] (M = 128 throughout):
// S = [Q_A; Q_B] [K_jA; K_jB]^T (N = 128; A's rows keep columns 0-63, B's
// 64-127; dense mode, where both blocks share K_j: N = 64) into one TMEM S
// buffer; the softmax reads its row's 64 scores and writes P into the
// block-diagonal P tile [128 rows][128 keys] (the other key half of a row stays
// zero); O += P [V_jA; V_jB] (K = 128 keys, N = d). S(t+1) is issued as soon as
// the softmax has read S(t), before PV(t). O is rescaled in TMEM only when a
// row maximum grows by more than 2^8 (the exponent headroom of bf16 P and fp32
// O). G += phi(K_j)^T V_j (M=d, N=d) over
// E_i: for the critical blocks right after PV(t) on the V tile already
// resident (bf16, d = 128), for the others in phase 2. Epilogue: phi(Q_i)
// (precomputed, loaded over Q_i) dotted with Z_i (precomputed) gives the
// denominator; H_i = H_tot - G in bf16 -> shared memory, num = [phi(Q_A);
// phi(Q_B)] H_X for X = A, B (M = 128, the rows of block X kept), SLA's
// Y = O^l W as one M = 128 product.
//
// Every wait is bounded (about 2 s); an expired wait sets the device status
// word to kDevTimeout and makes every later wait of the CTA return at once,
// so the kernel always terminates.
#include <string.h>

#include "tc_util.cuh"

namespace sla {

using namespace tc;

struct TcMaps {
  CUtensorMap q, k, v, phik, w, phiq, o;
  CUtensorMap ht;  // H_tot in bf16, [BH][d][d] (d = 128)
  CUtensorMap qc, kc, vc;  // INT8 Q, K and e4m3 V codes (quantised sparse branch)
};

// Pair tiles: the 64 rows of block A followed by the 64 rows of block B (or
// key blocks j_A, j_B), in 64-column SW128 sub-tiles of 128 rows x 128 B.
template <int D>
struct TcCfg {
  static constexpr int kSub = D / 64;          // 64-column sub-tiles of a row
  static constexpr int kTile = 64 * D * 2;     // bytes of a 64 x D bf16 tile
  static constexpr int kSubS = 128 * 128;      // bytes of one 128-row sub-tile
  static constexpr int kHalf = 64 * 128;       // offset of the B rows inside a sub-tile
  static constexpr int kNK = D == 128 ? 3 : 2; // K-ring slots (K pair | phi(K) pair)
  static constexpr int kNV = 2;                // V-ring slots (V pair)
  static constexpr int kPair = kSub * kSubS;   // bytes of one ring slot (= 2 kTile)
  static constexpr int oQ = 0;                 // Q pair tile (later phi(Q))
  static constexpr int oP = kPair;             // P: [128 rows][128 keys] bf16, two 64-key sub-tiles
  static constexpr int oK = oP + 2 * kSubS;
  static constexpr int oV = oK + kNK * kPair;
  static constexpr int kBytes = oV + kNV * kPair;
  // epilogue tiles reuse the rings once every loop product has completed
  static constexpr int kMat = D * D * 2;       // D x D bf16
  static constexpr int oHA = oK, oHB = oK + kMat, oW = oK + 2 * kMat;
  static constexpr int oOl = oK + 3 * kMat;    // O^l pair tile
  static_assert(oOl + kPair <= kBytes, "epilogue tiles must fit in the rings");
  // TMEM columns (fp32); row i of the pair in lane i
  static constexpr int cS = 0;                 // S: [128 rows][128 keys] (dense: 64)
  static constexpr int cO = 128;               // O: D columns
  static constexpr int cG = 128 + D;           // G_A (D=128: G_B at cG + 128; D=64: M=64 halves)
  static constexpr int cNumA = 0;              // num of block A (over S, after the loop)
  // d = 128: phi(Q) H_tot over S, phi(Q) (-G_A) over G_A, phi(Q) (-G_B) over G_B
  static constexpr int cT = 0, cNegA = cG, cNegB = cG + 128;
  static constexpr int cNumB = D == 128 ? cG : 64;        // num of block B (over G_A / S)
  static constexpr int cY = D == 128 ? cG + 128 : cG;     // Y = O^l W (over G_B / G)
  static constexpr uint32_t kTmemCols = D == 128 ? 512 : 256;
};

enum Bar {
  bQFull = 0,
  bKFull0, bKFull1, bKFull2, bKEmpty0, bKEmpty1, bKEmpty2, bKDone0, bKDone1, bKDone2,
  bVFull0, bVFull1, bVEmpty0, bVEmpty1,
  bSFull, bSFree, bPFull, bPvDone,
  bTailDone, bHiFull, bNumFull, bWFull, bOlFull, bYFull, bDrain, bQFree, bPhiQFull, bHtFull, kNumBars
};

// QNT: the sparse branch on the quantised forms (SLA2 article, quantisation
// paragraphs: Q, K, P, V go to low-bit values with a scale before the
// products and are restored after). S = Qc Kc^T on kind::i8 (int32 in TMEM),
// scaled by s_q,i s_k,j / sqrt(d); P~ = 2^(x - m) in fp32 (x = S log2 e), the
// row sum l uses P~; P enters PV as e4m3(P~ r_j 2^4) with r_j = s_v,j / max_j
// s_v,j (each key block's V scale folded into P); O^s = (sum P_q V_c) max s_v
// / 2^4 / l. m is an integer running row max raised lazily: P~ <= 2^kLazy =
// 2^4, so P~ r_j 2^4 <= 2^8 stays inside e4m3's range (448), and since m is
// an integer the codes are the row-max-rounded-up codes e4m3(P~ r_j 2^8)
// shifted by a power of two. The linear branch and the epilogue stay bf16
// (phi(Q) from the bf16 Q tile).
template <int D, int MODE, bool QNT>
__global__ void __launch_bounds__(192, 1) attn_tc_kernel(const __grid_constant__ TcMaps maps,
                                                         const AttnArgs a) {
  using C = TcCfg<D>;
  static_assert(!QNT || D == 128, "the quantised branch is built for d = 128");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float zs[2][D];
  // quantised branch: per-step key-block scale and V-scale ratio, 32-step window
  __shared__ float qwin_k[2][32], qwin_r[2][32];
  __shared__ float qred[4];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, h = bh % a.H;
  const int N = a.N, Nb = a.Nb;
  const int iA = 2 * blockIdx.x;
  const bool validB = iA + 1 < Nb;
  const int iB = validB ? iA + 1 : iA;
  constexpr bool dense = MODE == kModeDense;
  // lazy online softmax: the running max m (log2 units) is raised only when a
  // row's block max exceeds it by more than kLazy, so P~ <= 2^kLazy; the
  // quantised P is P~ r_j kPMul with kPMul = 2^(8 - kLazy) <= 2^8 < 448
  constexpr float kLazy = QNT ? 4.0f : 8.0f;
  constexpr float kPMul = QNT ? 16.0f : 1.0f;
  const int nA = dense ? Nb : a.kc;
  const bool has_marg = !dense && (a.kc + a.kn < Nb);
  const int nE = a.kc + a.kn;
  // merged mode (bf16, d = 128): the excluded-block products of the critical
  // blocks run in phase 1 on the V tiles already resident, phi(K_j) being
  // loaded into K_j's slot once S has read it; phase 2 then covers the
  // negligible blocks only. The quantised branch keeps V as e4m3 codes in
  // phase 1 and so takes every excluded block in phase 2.
  constexpr bool kMergeCapable = !QNT && MODE != kModeDense && D == 128;
  // d = 128: the linear numerator is phi(Q) H_tot (H_tot loaded as a bf16 tile)
  // plus phi(Q) (-G_X); d = 64 forms H_X = H_tot - G_X from the fp32 H_tot
  constexpr bool kHtTile = D == 128 && MODE != kModeDense;
  const bool merge = kMergeCapable && has_marg;
  // phi(Q) and Z_i precomputed (loaded) rather than formed in the epilogue
  const bool pre = has_marg && a.phiq != nullptr;
  // quantised branch with a marginal set: phase 1's code tiles fill half of
  // each ring slot, so every phase-1 step also carries one excluded block's
  // phi(K) and V (bf16) in the other halves and its G product (block A's
  // u-th excluded block on even steps, block B's on odd steps); phase 2 then
  // takes the excluded blocks from index `carried` on
  const bool hmerge = QNT && has_marg;
  const int carried = hmerge ? nA / 2 : 0;
  const int nP2 = has_marg ? (merge ? a.kn : nE - carried) : 0;  // phase-2 ring steps
  const int nTot = nA + nP2;                            // ring steps: phase 1 then phase 2
  const bool use_y = MODE == kModeSLA && a.w_proj != nullptr && has_marg;
  const int32_t* critA = a.crit + (size_t(bh) * Nb + iA) * a.kc;
  const int32_t* critB = a.crit + (size_t(bh) * Nb + iB) * a.kc;
  const int kn_stride = a.kn > 0 ? a.kn : 1;
  const int32_t* negA = a.neg + (size_t(bh) * Nb + iA) * kn_stride;
  const int32_t* negB = a.neg + (size_t(bh) * Nb + iB) * kn_stride;
  volatile int* abort_flag = &abort_sh;

  auto checked = [&](int j) {
    if (j < 0 || j >= Nb) {
      if (a.status) atomicExch(a.status, kDevBadIndex);
      j = j < 0 ? 0 : Nb - 1;
    }
    return j;
  };
  // key block of ring step T for block A (X = 0) or B (X = 1)
  // u-th excluded block (the critical ones, then the negligible ones)
  auto excl_block = [&](int X, int u) {
    const int32_t* cl = X ? critB : critA;
    const int32_t* nl = X ? negB : negA;
    return checked(u < a.kc ? cl[u] : nl[u - a.kc]);
  };
  auto step_block = [&](int X, int T) {
    if (dense) return T;
    if (T < nA) return checked((X ? critB : critA)[T]);
    return excl_block(X, T - nA + (merge ? a.kc : carried));
  };
  auto bar = [&](int b) { return smem_u32(&bars[b]); };
  auto wait = [&](int b, uint32_t parity) { return mbar_wait(bar(b), parity, abort_flag, a.status); };
  // reconverge the warp after a wait, before warp-collective tcgen05 loads / stores
  auto wait_w = [&](int b, uint32_t parity) {
    const bool ok = wait(b, parity);
    __syncwarp();
    return ok;
  };
  // bounded wait that ignores the abort flag: in-flight copies / MMAs must land before exit
  int no_abort = 0;
  auto wait_drain = [&](int b, uint32_t parity) {
    return mbar_wait(bar(b), parity, reinterpret_cast<volatile int*>(&no_abort), a.status);
  };

  const uint32_t sb = smem_u32(smem);
  const uint32_t sQ = sb + C::oQ, sP = sb + C::oP;
  const uint32_t sK = sb + C::oK, sV = sb + C::oV;
  const uint32_t sHA = sb + C::oHA, sHB = sb + C::oHB, sW = sb + C::oW;
  const uint32_t sOl = sb + C::oOl;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(bar(bQFull), 1);
    for (int s = 0; s < C::kNK; ++s) {
      mbar_init(bar(bKFull0 + s), 1);
      mbar_init(bar(bKEmpty0 + s), 1);
      mbar_init(bar(bKDone0 + s), 1);
    }
    for (int s = 0; s < C::kNV; ++s) {
      mbar_init(bar(bVFull0 + s), 1);
      mbar_init(bar(bVEmpty0 + s), 1);
    }
    mbar_init(bar(bSFull), 1);
    mbar_init(bar(bSFree), 128);
    mbar_init(bar(bPFull), 128);
    mbar_init(bar(bPvDone), 1);
    mbar_init(bar(bTailDone), 1);
    mbar_init(bar(bHiFull), 1);
    mbar_init(bar(bNumFull), 1);
    mbar_init(bar(bWFull), 1);
    mbar_init(bar(bOlFull), 1);
    mbar_init(bar(bYFull), 1);
    mbar_init(bar(bDrain), 1);
    mbar_init(bar(bQFree), 1);
    mbar_init(bar(bPhiQFull), 1);
    mbar_init(bar(bHtFull), 1);
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(smem_u32(&tmem_base_sh), C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tmem_base_sh;

  if (warp == 4) {
    // ------------------------------ TMA producer ------------------------------
    // The whole warp walks the steps; lane i prefetches the block indices of
    // 32 consecutive steps and lane 0 issues the copies.
    if (lane == 0) {
      prefetch_tmap(&maps.q);
      prefetch_tmap(&maps.k);
      prefetch_tmap(&maps.v);
      if (has_marg) {
        prefetch_tmap(&maps.phik);
        prefetch_tmap(&maps.phiq);
      }
      if constexpr (QNT) {  // INT8 Q codes: one 64 x 128-byte box per block
        mbar_expect_tx(bar(bQFull), 2 * 8192);
        tma_load_3d(sQ, &maps.qc, bar(bQFull), 0, iA * 64, bh);
        tma_load_3d(sQ + C::kHalf, &maps.qc, bar(bQFull), 0, iB * 64, bh);
      } else {
        mbar_expect_tx(bar(bQFull), 2 * C::kTile);
        for (int s = 0; s < C::kSub; ++s) {
          tma_load_3d(sQ + s * C::kSubS, &maps.q, bar(bQFull), s * 64, iA * 64, bh);
          tma_load_3d(sQ + s * C::kSubS + C::kHalf, &maps.q, bar(bQFull), s * 64, iB * 64, bh);
        }
      }
    }
    // bytes per ring step; dense mode loads one shared tile per step, the
    // quantised phase 1 one 8 KB code tile per block
    const int tileBytes = dense ? C::kTile : 2 * C::kTile;
    // Abort safety: a copy is issued only after its slot's release was
    // observed with no abort raised, so every slot has at most one copy in
    // flight; once a wait fails or the abort flag is up, no further copy is
    // issued. Before the warp leaves it waits (bounded, ignoring the abort
    // flag) for the last copy of every slot it filled, so no TMA write to
    // shared memory is still pending when the CTA exits.
    bool stop = false;
    auto pwait = [&](int b, uint32_t parity) {
      const bool ok = !stop && wait(b, parity) && *abort_flag == 0;
      stop = !__all_sync(0xffffffffu, ok);
      return !stop;
    };
    uint32_t kpar = 0, kany = 0;  // per K slot: parity of its next fill; slots filled at least once
    uint32_t vpar = 0, vany = 0;  // same for the V slots
    auto k_filled = [&](int st) {
      kany |= 1u << st;
      kpar ^= 1u << st;
    };
    auto v_filled = [&](int st) {
      vany |= 1u << st;
      vpar ^= 1u << st;
    };
    // phi(Q) (precomputed) over the Q or Q-code tiles once the last S product
    // has read them: the epilogue's phi(Q) H_i and phi(Q) Z_i operand
    bool phiq_issued = false;
    auto load_phiq = [&]() {
      if (!pwait(bQFree, 0)) return;
      if (lane == 0) {
        mbar_expect_tx(bar(bPhiQFull), 2 * C::kTile);
        for (int s = 0; s < C::kSub; ++s) {
          tma_load_3d(sQ + s * C::kSubS, &maps.phiq, bar(bPhiQFull), s * 64, iA * 64, bh);
          tma_load_3d(sQ + s * C::kSubS + C::kHalf, &maps.phiq, bar(bPhiQFull), s * 64, iB * 64, bh);
        }
      }
      phiq_issued = true;
      __syncwarp();
    };
    const int codeBytes = 2 * 8192;
    constexpr int lag = C::kNK - C::kNV;  // K copies run this many steps ahead of V copies
    int kA_reg = 0, kB_reg = 0;           // indices of the current 32-step window (K side)
    int vA_reg = 0, vB_reg = 0;           // indices of the window the V side reads
    int kH_reg = 0, vH_reg = 0;           // hmerge: the excluded block each phase-1 step carries
    auto carried_block = [&](int T) { return excl_block(T & 1, T >> 1); };
    if (!merge) {
      for (int T = 0; T < nTot + lag && !stop; ++T) {
        const int TK = T, TV = T - lag;
        if ((TK & 31) == 0 && TK < nTot) {
          const int Ti = TK + lane;
          kA_reg = Ti < nTot ? step_block(0, Ti) : 0;
          kB_reg = Ti < nTot ? step_block(1, Ti) : 0;
          kH_reg = Ti < 2 * carried ? carried_block(Ti) : 0;
        }
        if (TV >= 0 && (TV & 31) == 0 && TV < nTot) {
          const int Ti = TV + lane;
          vA_reg = Ti < nTot ? step_block(0, Ti) : 0;
          vB_reg = Ti < nTot ? step_block(1, Ti) : 0;
          vH_reg = Ti < 2 * carried ? carried_block(Ti) : 0;
        }
        if (TK < nTot) {
          const int jA = __shfl_sync(0xffffffffu, kA_reg, TK & 31);
          const int jB = __shfl_sync(0xffffffffu, kB_reg, TK & 31);
          const int jH = __shfl_sync(0xffffffffu, kH_reg, TK & 31);
          const int st = TK % C::kNK;
          if (!pwait(bKEmpty0 + st, ((TK / C::kNK) & 1) ^ 1)) break;
          if (lane == 0) {
            const uint32_t slot = sK + st * C::kPair;
            if (QNT && TK < nA) {
              const bool carry = TK < 2 * carried;
              mbar_expect_tx(bar(bKFull0 + st), codeBytes + (carry ? C::kTile : 0));
              tma_load_3d(slot, &maps.kc, bar(bKFull0 + st), 0, jA * 64, bh);
              tma_load_3d(slot + C::kHalf, &maps.kc, bar(bKFull0 + st), 0, jB * 64, bh);
              if (carry)  // phi(K) of the carried block in the slot's other half
                for (int s = 0; s < C::kSub; ++s)
                  tma_load_3d(slot + C::kSubS + s * 8192, &maps.phik, bar(bKFull0 + st), s * 64, jH * 64, bh);
            } else {
              const CUtensorMap* km = TK < nA ? &maps.k : &maps.phik;
              mbar_expect_tx(bar(bKFull0 + st), tileBytes);
              for (int s = 0; s < C::kSub; ++s) {
                tma_load_3d(slot + s * C::kSubS, km, bar(bKFull0 + st), s * 64, jA * 64, bh);
                if (!dense)
                  tma_load_3d(slot + s * C::kSubS + C::kHalf, km, bar(bKFull0 + st), s * 64, jB * 64, bh);
              }
            }
          }
          k_filled(st);
          __syncwarp();
        }
        if (TV >= 0 && TV < nTot) {
          const int jA = __shfl_sync(0xffffffffu, vA_reg, TV & 31);
          const int jB = __shfl_sync(0xffffffffu, vB_reg, TV & 31);
          const int jH = __shfl_sync(0xffffffffu, vH_reg, TV & 31);
          const int st = TV % C::kNV;
          if (!pwait(bVEmpty0 + st, ((TV / C::kNV) & 1) ^ 1)) break;
          if (lane == 0) {
            const uint32_t slot = sV + st * C::kPair;
            if (QNT && TV < nA) {
              const bool carry = TV < 2 * carried;
              mbar_expect_tx(bar(bVFull0 + st), codeBytes + (carry ? C::kTile : 0));
              tma_load_3d(slot, &maps.vc, bar(bVFull0 + st), 0, jA * 64, bh);
              tma_load_3d(slot + C::kHalf, &maps.vc, bar(bVFull0 + st), 0, jB * 64, bh);
              if (carry)  // V (bf16) of the carried block in the slot's other half
                for (int s = 0; s < C::kSub; ++s)
                  tma_load_3d(slot + C::kSubS + s * 8192, &maps.v, bar(bVFull0 + st), s * 64, jH * 64, bh);
            } else {
              mbar_expect_tx(bar(bVFull0 + st), tileBytes);
              for (int s = 0; s < C::kSub; ++s) {
                tma_load_3d(slot + s * C::kSubS, &maps.v, bar(bVFull0 + st), s * 64, jA * 64, bh);
                if (!dense)
                  tma_load_3d(slot + s * C::kSubS + C::kHalf, &maps.v, bar(bVFull0 + st), s * 64, jB * 64, bh);
              }
            }
          }
          v_filled(st);
          __syncwarp();
        }
      }
    } else {
      // Merged mode. Step t: K(t); then, one step behind, V(t-1) and phi(K)(t-1)
      // into K(t-1)'s slot once S(t-1) has read it (KDone). Phase 2: phi(K) and
      // V of the negligible blocks. A K slot is filled twice per phase-1 step,
      // so its barrier phases are tracked per slot in bit masks.
      auto load_pair = [&](uint32_t slot, const CUtensorMap* m, uint32_t fb, int jA, int jB) {
        mbar_expect_tx(fb, 2 * C::kTile);
        for (int s = 0; s < C::kSub; ++s) {
          tma_load_3d(slot + s * C::kSubS, m, fb, s * 64, jA * 64, bh);
          tma_load_3d(slot + s * C::kSubS + C::kHalf, m, fb, s * 64, jB * 64, bh);
        }
      };
      uint32_t pe = (1u << C::kNK) - 1;  // KEmpty parity per slot (a slot's first fill passes)
      uint32_t pd = 0;                   // KDone parity per slot
      for (int t = 0; t <= nA && !stop; ++t) {
        if ((t & 31) == 0 && t < nA) {
          const int Ti = t + lane;
          kA_reg = Ti < nA ? step_block(0, Ti) : 0;
          kB_reg = Ti < nA ? step_block(1, Ti) : 0;
        }
        if (t >= 1 && ((t - 1) & 31) == 0) {
          const int Ti = t - 1 + lane;
          vA_reg = Ti < nA ? step_block(0, Ti) : 0;
          vB_reg = Ti < nA ? step_block(1, Ti) : 0;
        }
        if (t < nA) {  // K(t)
          const int jA = __shfl_sync(0xffffffffu, kA_reg, t & 31);
          const int jB = __shfl_sync(0xffffffffu, kB_reg, t & 31);
          const int st = t % C::kNK;
          if (!pwait(bKEmpty0 + st, (pe >> st) & 1u)) break;
          pe ^= 1u << st;
          if (lane == 0) load_pair(sK + st * C::kPair, &maps.k, bar(bKFull0 + st), jA, jB);
          k_filled(st);
          __syncwarp();
        }
        if (t >= 1) {  // V(t-1), then phi(K)(t-1)
          const int u = t - 1;
          const int jA = __shfl_sync(0xffffffffu, vA_reg, u & 31);
          const int jB = __shfl_sync(0xffffffffu, vB_reg, u & 31);
          const int sv = u % C::kNV, st = u % C::kNK;
          if (!pwait(bVEmpty0 + sv, ((u / C::kNV) & 1) ^ 1)) break;
          if (lane == 0) load_pair(sV + sv * C::kPair, &maps.v, bar(bVFull0 + sv), jA, jB);
          v_filled(sv);
          __syncwarp();
          if (!pwait(bKDone0 + st, (pd >> st) & 1u)) break;
          pd ^= 1u << st;
          if (lane == 0) load_pair(sK + st * C::kPair, &maps.phik, bar(bKFull0 + st), jA, jB);
          k_filled(st);
          __syncwarp();
        }
      }
      if (pre && !stop) load_phiq();  // S(nA-1) has completed: phi(K)(nA-1) waited for it
      for (int u = 0; u < nP2 && !stop; ++u) {  // the negligible blocks
        const int T = nA + u;
        if ((u & 31) == 0) {
          const int Ti = T + lane;
          kA_reg = Ti < nTot ? step_block(0, Ti) : 0;
          kB_reg = Ti < nTot ? step_block(1, Ti) : 0;
        }
        const int jA = __shfl_sync(0xffffffffu, kA_reg, u & 31);
        const int jB = __shfl_sync(0xffffffffu, kB_reg, u & 31);
        const int st = T % C::kNK, sv = T % C::kNV;
        if (!pwait(bKEmpty0 + st, (pe >> st) & 1u)) break;
        pe ^= 1u << st;
        if (lane == 0) load_pair(sK + st * C::kPair, &maps.phik, bar(bKFull0 + st), jA, jB);
        k_filled(st);
        __syncwarp();
        if (!pwait(bVEmpty0 + sv, ((T / C::kNV) & 1) ^ 1)) break;
        if (lane == 0) load_pair(sV + sv * C::kPair, &maps.v, bar(bVFull0 + sv), jA, jB);
        v_filled(sv);
        __syncwarp();
      }
    }
    if (pre && !merge && !stop) load_phiq();
    // d = 128: H_tot (bf16) into the V slot the next fill would take, once the
    // products that read that slot's last V have completed
    bool ht_issued = false;
    if (kHtTile && has_marg && !stop) {
      const int sv = nTot % C::kNV;
      if (pwait(bVEmpty0 + sv, ((nTot / C::kNV) & 1) ^ 1)) {
        if (lane == 0) {
          mbar_expect_tx(bar(bHtFull), C::kMat);
          tma_load_3d(sV + sv * C::kPair, &maps.ht, bar(bHtFull), 0, 0, bh);
          tma_load_3d(sV + sv * C::kPair + D * 128, &maps.ht, bar(bHtFull), 64, 0, bh);
        }
        ht_issued = true;
      }
      __syncwarp();
    }
    bool w_issued = false;
    if (use_y && pwait(bTailDone, 0)) {  // W reuses the rings once every loop product has completed
      if (lane == 0) {
        mbar_expect_tx(bar(bWFull), C::kMat);
        for (int s = 0; s < C::kSub; ++s) tma_load_2d(sW + s * (D * 128), &maps.w, bar(bWFull), s * 64, 0);
      }
      w_issued = true;
    }
    // drain: the last copy of every slot, Q, phi(Q) and W have landed
    if (lane == 0) {
      wait_drain(bQFull, 0);
      for (int st = 0; st < C::kNK; ++st)
        if ((kany >> st) & 1u) wait_drain(bKFull0 + st, ((kpar >> st) & 1u) ^ 1u);
      for (int st = 0; st < C::kNV; ++st)
        if ((vany >> st) & 1u) wait_drain(bVFull0 + st, ((vpar >> st) & 1u) ^ 1u);
      if (phiq_issued) wait_drain(bPhiQFull, 0);
      if (ht_issued) wait_drain(bHtFull, 0);
      if (w_issued) wait_drain(bWFull, 0);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------ MMA issuer ------------------------------
    // The whole warp walks the loop (warp-uniform descriptors); the MMA and
    // commit helpers issue from one elected lane.
    {
      // S, PV, num and Y run at M = 128 over the row pair (A rows, then B rows)
      constexpr uint32_t idS = idesc_bf16(128, dense ? 64 : 128, 0, 0);
      constexpr uint32_t idPV = idesc_bf16(128, D, 0, 1);
      constexpr uint32_t idG = idesc_bf16(D, D, 1, 1);
      constexpr uint32_t idN = idesc_bf16(128, D, 0, 1);
      constexpr uint32_t laneB = 16u << 16;  // D=64: G_B's M=64 accumulator starts at lane 16
      wait_w(bQFull, 0);
      tc_fence_after();
      const uint32_t gA = tb + C::cG;
      const uint32_t gB = D == 128 ? tb + C::cG + 128 : tb + laneB + C::cG;
      auto issue_pv = [&](int tp) {
        const int stv = tp % C::kNV;
        wait_w(bVFull0 + stv, (tp / C::kNV) & 1);
        wait_w(bPFull, tp & 1);
        tc_fence_after();
        const uint32_t vslot = sV + stv * C::kPair;
        if constexpr (QNT) {
          // A = P e4m3 [128 rows][128 keys] (block diagonal: A rows over j_A's
          // keys, B rows over j_B's), SW128; B = V codes [128 keys][128 dims]
          // MN-major; K = 32 keys per instruction
          constexpr uint32_t idPV8 = idesc_e4m3(128, D, 0, 1);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t acc = (tp > 0 || k > 0) ? 1u : 0u;
            mma_e4m3(tb + C::cO, sdesc(sP + k * 32, 16, 1024), sdesc(vslot + k * 4096, C::kSubS, 1024), idPV8, acc);
          }
        } else {
          // A = P bf16 [128 rows][128 keys] block diagonal (dense: [128][64]),
          // B = V pair [128 keys][D] MN-major
          constexpr int nk = dense ? 4 : 8;
#pragma unroll
          for (int k = 0; k < nk; ++k) {
            const uint32_t acc = (tp > 0 || k > 0) ? 1u : 0u;
            mma_bf16(tb + C::cO, sdesc(sP + (k >> 2) * C::kSubS + (k & 3) * 32, 16, 1024),
                     sdesc(vslot + k * 2048, C::kSubS, 1024), idPV, acc);
          }
        }
        mma_commit(bar(bPvDone));
        if (hmerge) {
          // the carried block's G += phi(K_j)^T V_j from the slots' other
          // halves (64 tokens, M = N = D, MN-major, 64-column boxes 8 KB apart),
          // then both slots are free
          const int stk = tp % C::kNK;
          if (tp < 2 * carried) {
            const uint32_t kh = sK + stk * C::kPair + C::kSubS, vh = vslot + C::kSubS;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16((tp & 1) ? gB : gA, sdesc(kh + k * 2048, 8192, 1024), sdesc(vh + k * 2048, 8192, 1024),
                       idesc_bf16(D, D, 1, 1), (tp >= 2 || k > 0) ? 1u : 0u);
          }
          mma_commit(bar(bKEmpty0 + stk));
        }
        if (!merge) mma_commit(bar(bVEmpty0 + stv));  // merged: released after G
      };
      // G += phi(K_j)^T V_j for both blocks (M = N = D, MN-major operands; the
      // j_B rows sit kHalf into each sub-tile)
      auto issue_g = [&](uint32_t kslot, uint32_t vslot, bool first) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t acc = (!first || k > 0) ? 1u : 0u;
          mma_bf16(gA, sdesc(kslot + k * 2048, C::kSubS, 1024), sdesc(vslot + k * 2048, C::kSubS, 1024), idG, acc);
          mma_bf16(gB, sdesc(kslot + C::kHalf + k * 2048, C::kSubS, 1024),
                   sdesc(vslot + C::kHalf + k * 2048, C::kSubS, 1024), idG, acc);
        }
      };
      uint32_t kf = 0;  // KFull parity per slot
      auto wait_kfull = [&](int stk) {
        wait_w(bKFull0 + stk, (kf >> stk) & 1u);
        kf ^= 1u << stk;
      };
      // merged mode: G for critical step tp, after PV(tp), on phi(K)(tp) and V(tp)
      auto issue_g1 = [&](int tp) {
        const int stk = tp % C::kNK, stv = tp % C::kNV;
        wait_kfull(stk);
        tc_fence_after();
        issue_g(sK + stk * C::kPair, sV + stv * C::kPair, tp == 0);
        mma_commit(bar(bKEmpty0 + stk));
        mma_commit(bar(bVEmpty0 + stv));
      };
      for (int t = 0; t < nA; ++t) {
        const int stk = t % C::kNK;
        wait_kfull(stk);
        wait_w(bSFree, (t & 1) ^ 1);  // the softmax has read S(t-1)
        tc_fence_after();
        const uint32_t kslot = sK + stk * C::kPair;
        if constexpr (QNT) {
          // INT8 codes, one 128-byte swizzled row per token; K = 32 per instruction
          constexpr uint32_t idS8 = idesc_s8(128, 128);
#pragma unroll
          for (int k = 0; k < D / 32; ++k)
            mma_s8(tb + C::cS, sdesc(sQ + k * 32, 16, 1024), sdesc(kslot + k * 32, 16, 1024), idS8, k > 0);
        } else {
          // [Q_A; Q_B] [K_jA; K_jB]^T (dense: [Q_A; Q_B] K_j^T); the A rows use
          // columns 0-63, the B rows 64-127
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * C::kSubS + (k & 3) * 32;
            mma_bf16(tb + C::cS, sdesc(sQ + off, 16, 1024), sdesc(kslot + off, 16, 1024), idS, k > 0);
          }
        }
        mma_commit(bar(bSFull));
        // merged: phi(K) refills the slot; hmerge: the slot is released after
        // the carried block's G, with its PV
        if (!hmerge) mma_commit(bar(merge ? bKDone0 + stk : bKEmpty0 + stk));
        if (pre && t == nA - 1) mma_commit(bar(bQFree));          // Q tiles free for phi(Q)
        if (t > 0) {
          issue_pv(t - 1);
          if (merge) issue_g1(t - 1);
        }
      }
      if (nA > 0) {
        issue_pv(nA - 1);
        if (merge) issue_g1(nA - 1);
      }
      for (int u = 0; u < nP2; ++u) {  // phase 2
        const int T = nA + u, stk = T % C::kNK, stv = T % C::kNV;
        wait_kfull(stk);
        wait_w(bVFull0 + stv, (T / C::kNV) & 1);
        tc_fence_after();
        issue_g(sK + stk * C::kPair, sV + stv * C::kPair, !merge && carried == 0 && u == 0);
        mma_commit(bar(bKEmpty0 + stk));
        mma_commit(bar(bVEmpty0 + stv));
      }
      mma_commit(bar(bTailDone));
      if (has_marg) {
        wait_w(bHiFull, 0);
        if constexpr (kHtTile) wait_w(bHtFull, 0);
        tc_fence_after();
        if constexpr (kHtTile) {
          // T = [phi(Q_A); phi(Q_B)] H_tot (both blocks' rows kept) and
          // [phi(Q_A); phi(Q_B)] (-G_X) for X = A, B (the rows of block X kept)
          const uint32_t sHt = sV + (nTot % C::kNV) * C::kPair;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * C::kSubS + (k & 3) * 32;
            mma_bf16(tb + C::cT, sdesc(sQ + off, 16, 1024), sdesc(sHt + k * 2048, D * 128, 1024), idN, k > 0);
            mma_bf16(tb + C::cNegA, sdesc(sQ + off, 16, 1024), sdesc(sHA + k * 2048, D * 128, 1024), idN, k > 0);
            mma_bf16(tb + C::cNegB, sdesc(sQ + off, 16, 1024), sdesc(sHB + k * 2048, D * 128, 1024), idN, k > 0);
          }
        } else {
          // [phi(Q_A); phi(Q_B)] H_A and [phi(Q_A); phi(Q_B)] H_B: the A rows of
          // the first and the B rows of the second are kept
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * C::kSubS + (k & 3) * 32;
            mma_bf16(tb + C::cNumA, sdesc(sQ + off, 16, 1024), sdesc(sHA + k * 2048, D * 128, 1024), idN, k > 0);
            mma_bf16(tb + C::cNumB, sdesc(sQ + off, 16, 1024), sdesc(sHB + k * 2048, D * 128, 1024), idN, k > 0);
          }
        }
        mma_commit(bar(bNumFull));
      }
      if (use_y) {
        wait_w(bWFull, 0);
        wait_w(bOlFull, 0);
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * C::kSubS + (k & 3) * 32;
          mma_bf16(tb + C::cY, sdesc(sOl + off, 16, 1024), sdesc(sW + k * 2048, D * 128, 1024), idN, k > 0);
        }
        mma_commit(bar(bYFull));
      }
      // every MMA of this thread has completed before TMEM is released
      mma_commit(bar(bDrain));
      wait_drain(bDrain, 0);
      __syncwarp();
    }
  } else {
    // --------------------------- softmax / epilogue ---------------------------
    const int tid = threadIdx.x;  // 0..127: row of the pair = TMEM lane
    const bool isB = tid >= 64;   // warps 2-3
    const int blk = isB ? iB : iA;
    const uint32_t tq = tb + (uint32_t(32 * warp) << 16);  // this warp's TMEM lane quarter
    // this row's S columns and its P row (bf16: the 64-key sub-tile of its key
    // block; e4m3: its half of a 128-byte row); the other half of the row stays zero
    const int scol = dense ? 0 : (isB ? 64 : 0);
    unsigned char* Prow = smem + C::oP + (QNT ? 0 : (dense || !isB ? 0 : C::kSubS)) + tid * 128;
    if (!dense) {
      if constexpr (QNT) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(Prow + (uint32_t((c + (isB ? 0 : 4)) ^ (tid & 7)) << 4)) = make_uint4(0, 0, 0, 0);
      } else {
        unsigned char* other = smem + C::oP + (isB ? 0 : C::kSubS) + tid * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(other + (c << 4)) = make_uint4(0, 0, 0, 0);
      }
    }
    const float sl2 = a.scale_log2;
    // Only the block holding the last (partial) rows of the sequence has pad
    // keys; the lists are ascending, so it can only be the last step.
    const int jlast = dense ? Nb - 1 : checked((isB ? critB : critA)[nA - 1]);
    const bool mask_last = jlast * 64 + 64 > N;
    float m = -INFINITY, l = 0.0f;
    // precomputed Z_i of blocks A and B, read now so that the epilogue does not wait for it
    float zpre[2] = {0.0f, 0.0f};
    if (pre) {
      const float* zia = a.zi + (size_t(bh) * Nb + iA) * D;
      const float* zib = a.zi + (size_t(bh) * Nb + iB) * D;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int e = tid + 128 * k;
        if (e < 2 * D) zpre[k] = (e < D ? zia : zib)[e % D];
      }
    }
    // quantised branch: the row's INT8 scale and the head's largest V scale
    float q_scale = 1.0f, sv_max = 1.0f;
    if constexpr (QNT) {
      const float* vs = a.vscale + size_t(bh) * Nb;
      float vm = 0.0f;
      for (int j = tid; j < Nb; j += 128) vm = fmaxf(vm, vs[j]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, off));
      if (lane == 0) qred[warp] = vm;
      named_bar(1, 128);
      sv_max = fmaxf(fmaxf(qred[0], qred[1]), fmaxf(qred[2], qred[3]));
      q_scale = a.qscale[size_t(bh) * Nb + blk];
    }

    for (int t = 0; t < nA; ++t) {
      if constexpr (QNT) {
        if ((t & 31) == 0) {  // scales of the next 32 steps
          named_bar(1, 128);
          const int T = t + tid;
          if (tid < 32 && T < nA) {
#pragma unroll
            for (int X = 0; X < 2; ++X) {
              const int j = step_block(X, T);
              qwin_k[X][tid] = a.kscale[size_t(bh) * Nb + j];
              qwin_r[X][tid] = a.vscale[size_t(bh) * Nb + j] / sv_max;
            }
          }
          named_bar(1, 128);
        }
      }
      wait_w(bSFull, t & 1);
      tc_fence_after();
      float s[64];
      {
        float lo[32], hi[32];
        tmem_ld32(tq + C::cS + scol, lo);
        tmem_ld32(tq + C::cS + scol + 32, hi);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = lo[i];
          s[32 + i] = hi[i];
        }
      }
      tc_fence_before();
      mbar_arrive(bar(bSFree));
      // scale of this step's scores into log2 units (quantised: int32 S times
      // s_q,i s_k,j)
      float cs = sl2;
      if constexpr (QNT) {
#pragma unroll
        for (int i = 0; i < 64; ++i) s[i] = float(__float_as_int(s[i]));
        cs = sl2 * q_scale * qwin_k[isB][t & 31];
      }
      if (t == nA - 1 && mask_last) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (jlast * 64 + i >= N) s[i] = -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) mx8[g] = s[g];
#pragma unroll
      for (int i = 8; i < 64; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], s[i]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * cs;
      // quantised: m is an integer, so P~ = 2^(x - m) differs from the
      // exact-max P~ by a power of two and its e4m3 codes are those of the
      // exact-max P~ shifted in exponent; every rescale is an exact 2^k
      if (t == 0) {
        m = QNT ? ceilf(mx) : mx;
      } else if (__any_sync(0xffffffffu, mx > m + kLazy)) {
        // some row of this warp grew by more than 2^kLazy: rescale the warp's O rows in TMEM
        // once PV(t-1) has landed in O
        wait_w(bPvDone, (t - 1) & 1);
        tc_fence_after();
        const float mnew = QNT ? ceilf(fmaxf(m, mx)) : fmaxf(m, mx);
        float corr;
        if constexpr (QNT) {
          const int k = int(m - mnew);  // <= 0
          corr = k < -126 ? 0.0f : __int_as_float((k + 127) << 23);
        } else {
          corr = ex2(m - mnew);
        }
        l *= corr;
        m = mnew;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(tq + C::cO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= corr;
          tmem_st32(tq + C::cO + c * 32, o);
        }
        tmem_wait_st();
      }
      uint32_t pk[32];
      float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      // quantised: P~ (V scale folded in) scaled by kPMul into e4m3
      const float pq_mul = QNT ? qwin_r[isB][t & 31] * kPMul : 1.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float p0 = ex2(fmaf(s[2 * i], cs, -m));
        const float p1 = ex2(fmaf(s[2 * i + 1], cs, -m));
        sum8[i & 7] += p0 + p1;
        pk[i] = QNT ? pack_e4m3x2(p0 * pq_mul, p1 * pq_mul) : pack_bf16(p0, p1);
      }
      l += ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
      // the P buffer is free once PV(t-1) has completed
      if (t >= 1) wait(bPvDone, (t - 1) & 1);
      if constexpr (QNT) {
        // e4m3 P: this row's 64 keys in its half of the 128-byte SW128 row
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(Prow + (uint32_t((c + (isB ? 4 : 0)) ^ (tid & 7)) << 4)) =
              make_uint4(pk[8 * c] | (pk[8 * c + 1] << 16), pk[8 * c + 2] | (pk[8 * c + 3] << 16),
                         pk[8 * c + 4] | (pk[8 * c + 5] << 16), pk[8 * c + 6] | (pk[8 * c + 7] << 16));
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(Prow + (uint32_t(c ^ (tid & 7)) << 4)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar(bPFull));
    }
    // final O: the last PV (and every earlier product) has completed
    wait_w(bPvDone, (nA - 1) & 1);
    tc_fence_after();
    // quantised: undo the kPMul P scale and the V-scale fold
    const float inv_l = (QNT ? sv_max * (1.0f / kPMul) : 1.0f) / l;

    float den = 1.0f;
    if (pre) {
      // Z_i of blocks A and B (precomputed, loaded before the loop), then
      // den = phi(Q_i) . Z_i from the phi(Q) tile the producer loads over Q
      // once the last S product is done
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int e = tid + 128 * k;
        if (e < 2 * D) zs[e / D][e % D] = zpre[k];
      }
      named_bar(1, 128);  // zs complete
      wait_w(bPhiQFull, 0);
      const unsigned char* Qt = smem + C::oQ;
      den = 0.0f;
#pragma unroll 4
      for (int c = 0; c < D / 8; ++c) {
        const uint4 raw = *reinterpret_cast<const uint4*>(Qt + (c >> 3) * C::kSubS + sw128_chunk(tid, c & 7));
        const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          den += bf16_lo(wv[e]) * zs[isB][8 * c + 2 * e] + bf16_hi(wv[e]) * zs[isB][8 * c + 2 * e + 1];
      }
    } else if (has_marg) {
      // Z_i = Z_tot - sum over the excluded blocks of z_j, blocks A and B.
      // Thread handles (X, c) for e = tid and tid + 128 < 2D; block indices are
      // fetched 32 at a time, one per lane, and broadcast.
      const float* zt = a.ztot + size_t(bh) * D;
      const float* zb = a.zblk + size_t(bh) * Nb * D;
      float z[2];
      int zc[2], zx[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int e = tid + 128 * k;
        zx[k] = e / D;
        zc[k] = e % D;
        z[k] = e < 2 * D ? zt[zc[k]] : 0.0f;
      }
      for (int u0 = 0; u0 < nE; u0 += 32) {
        const int uu = u0 + lane;
        const int myA = uu < nE ? excl_block(0, uu) : 0;
        const int myB = uu < nE ? excl_block(1, uu) : 0;
        const int cnt = min(32, nE - u0);
#pragma unroll 4
        for (int i = 0; i < cnt; ++i) {
          const int jA = __shfl_sync(0xffffffffu, myA, i);
          const int jB = __shfl_sync(0xffffffffu, myB, i);
#pragma unroll
          for (int k = 0; k < 2; ++k)
            if (tid + 128 * k < 2 * D) z[k] -= zb[size_t(zx[k] ? jB : jA) * D + zc[k]];
        }
      }
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (tid + 128 * k < 2 * D) zs[zx[k]][zc[k]] = z[k];
      // phi(Q) of this row, in place of the bf16 Q tile (K-major swizzled);
      // three passes over shared memory (max, sum, write) keep the row out of
      // registers
      unsigned char* Qt = smem + C::oQ;
      auto qchunk = [&](int c) -> uint4* {
        return reinterpret_cast<uint4*>(Qt + (c >> 3) * C::kSubS + sw128_chunk(tid, c & 7));
      };
      // phi = softmax over the row (max and sum passes first) or elu + 1
      // elementwise (qm = 0 and qinv = 1 are unused then)
      const bool elu1 = a.phi_elu1 != 0;
      float qm = -INFINITY, qinv = 1.0f;
      if (!elu1) {
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
          const uint4 raw = *qchunk(c);
          const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) qm = fmaxf(qm, fmaxf(bf16_lo(wv[e]), bf16_hi(wv[e])));
        }
        float qs = 0.0f;
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
          const uint4 raw = *qchunk(c);
          const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) qs += expf(bf16_lo(wv[e]) - qm) + expf(bf16_hi(wv[e]) - qm);
        }
        qinv = 1.0f / qs;
      }
      auto phi1 = [&](float x) { return elu1 ? (x > 0.0f ? x + 1.0f : expf(x)) : expf(x - qm) * qinv; };
      named_bar(1, 128);  // zs complete
      den = 0.0f;
#pragma unroll 4
      for (int c = 0; c < D / 8; ++c) {
        const uint4 raw = *qchunk(c);
        const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          pk[e] = pack_bf16(phi1(bf16_lo(wv[e])), phi1(bf16_hi(wv[e])));
          den += bf16_lo(pk[e]) * zs[isB][8 * c + 2 * e] + bf16_hi(pk[e]) * zs[isB][8 * c + 2 * e + 1];
        }
        *qchunk(c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
    if (has_marg && kHtTile) {
      // -G_A, -G_B -> bf16, MN-major tiles [D rows c][D cols e] (G row c =
      // TMEM lane c); the numerator is then phi(Q) H_tot + phi(Q) (-G_X)
      wait_w(bTailDone, 0);
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        float g[2][32];
        tmem_ld32(tq + C::cG + ch * 32, g[0]);
        tmem_ld32(tq + C::cG + 128 + ch * 32, g[1]);
        tmem_wait_ld();
#pragma unroll
        for (int X = 0; X < 2; ++X) {
          unsigned char* Hbase = smem + (X ? C::oHB : C::oHA);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const int e0 = ch * 32 + q8 * 8;
            const float* gx = g[X] + q8 * 8;
            const uint4 v = make_uint4(pack_bf16(-gx[0], -gx[1]), pack_bf16(-gx[2], -gx[3]),
                                       pack_bf16(-gx[4], -gx[5]), pack_bf16(-gx[6], -gx[7]));
            *reinterpret_cast<uint4*>(Hbase + (e0 >> 6) * (D * 128) + sw128_chunk(tid, (e0 & 63) >> 3)) = v;
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      named_bar(1, 128);
      if (tid == 0) mbar_arrive(bar(bHiFull));
      wait_w(bNumFull, 0);
      tc_fence_after();
    } else if (has_marg) {
      // H_i = H_tot - G_i -> bf16, MN-major tile [D rows c][D cols e]
      // D=128: G rows c = TMEM lanes (M = 128), G_A and G_B in separate columns;
      // D=64:  G_A rows in lanes 0-15 of each quarter, G_B in lanes 16-31.
      const int c = D == 128 ? tid : 16 * warp + (lane & 15);
      const bool g64B = lane >= 16;  // D=64: this lane holds G_B
      constexpr int kBlocksPerThread = D == 128 ? 2 : 1;
      const float* hrow = a.htot32 + size_t(bh) * D * D + size_t(c) * D;
      // H_tot row loads run one 32-column chunk ahead; chunk 0's before the
      // wait for the last G product
      float4 hv[8], hn[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) hv[q] = *reinterpret_cast<const float4*>(hrow + 4 * q);
      wait_w(bTailDone, 0);
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        if (ch + 1 < D / 32) {
#pragma unroll
          for (int q = 0; q < 8; ++q) hn[q] = *reinterpret_cast<const float4*>(hrow + (ch + 1) * 32 + 4 * q);
        }
        float g[kBlocksPerThread][32];
#pragma unroll
        for (int X = 0; X < kBlocksPerThread; ++X) tmem_ld32(tq + C::cG + (D == 128 ? X * 128 : 0) + ch * 32, g[X]);
        tmem_wait_ld();
#pragma unroll
        for (int X = 0; X < kBlocksPerThread; ++X) {
          const bool xb = D == 128 ? X == 1 : g64B;
          unsigned char* Hbase = smem + (xb ? C::oHB : C::oHA);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const int e0 = ch * 32 + q8 * 8;
            const float4 h0 = hv[2 * q8], h1 = hv[2 * q8 + 1];
            const float* gx = g[X] + q8 * 8;
            const uint4 v = make_uint4(pack_bf16(h0.x - gx[0], h0.y - gx[1]), pack_bf16(h0.z - gx[2], h0.w - gx[3]),
                                       pack_bf16(h1.x - gx[4], h1.y - gx[5]), pack_bf16(h1.z - gx[6], h1.w - gx[7]));
            *reinterpret_cast<uint4*>(Hbase + (e0 >> 6) * (D * 128) + sw128_chunk(c, (e0 & 63) >> 3)) = v;
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) hv[q] = hn[q];
      }
      fence_async_smem();
      tc_fence_before();
      named_bar(1, 128);
      if (tid == 0) mbar_arrive(bar(bHiFull));
      wait_w(bNumFull, 0);
      tc_fence_after();
    }

    const float alpha = MODE == kModeSLA2 ? a.alpha[h] : 0.0f;
    const float inv_den = 1.0f / den;
    // training forward: O^s, O^l, the row's log-normaliser and den, row by row
    const int grow = blk * 64 + (tid & 63);
    const bool srow = MODE != kModeDense && !QNT && a.save_os != nullptr && grow < N && (!isB || validB);
    const size_t sidx = size_t(bh) * (size_t(Nb) * 64) + grow;
    auto save_row = [&](__nv_bfloat16* dst, int ch, const float* v, float mul) {
      uint4* p = reinterpret_cast<uint4*>(dst + sidx * D + ch * 32);
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8)
        p[q8] = make_uint4(pack_bf16(v[8 * q8] * mul, v[8 * q8 + 1] * mul), pack_bf16(v[8 * q8 + 2] * mul, v[8 * q8 + 3] * mul),
                           pack_bf16(v[8 * q8 + 4] * mul, v[8 * q8 + 5] * mul), pack_bf16(v[8 * q8 + 6] * mul, v[8 * q8 + 7] * mul));
    };
    if (srow) {
      a.save_lse[sidx] = (m + log2f(l)) * 0.69314718055994531f;
      a.save_den[sidx] = has_marg ? den : 0.0f;
    }
    // this row's linear numerator, columns 32 ch .. 32 ch + 31
    auto load_num = [&](int ch, float (&x)[32]) {
      if constexpr (kHtTile) {
        float ng[32];
        tmem_ld32(tq + C::cT + ch * 32, x);
        tmem_ld32(tq + (isB ? C::cNegB : C::cNegA) + ch * 32, ng);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] += ng[i];
      } else {
        tmem_ld32(tq + (isB ? C::cNumB : C::cNumA) + ch * 32, x);
        tmem_wait_ld();
      }
    };
    // O is staged as a bf16 pair tile in the P region (free after the last PV)
    // and written by TMA; the tensor map's row extent N drops the pad rows
    unsigned char* Ot = smem + C::oP;
    if (use_y) {
      // O^l (bf16) -> K-major tile, then Y = O^l W on the tensor core
      unsigned char* Olt = smem + C::oOl;
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        float nm[32];
        load_num(ch, nm);
        if (srow) save_row(a.save_ol, ch, nm, inv_den);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const int e0 = ch * 32 + q8 * 8;
          const uint4 v = make_uint4(pack_bf16(nm[q8 * 8 + 0] * inv_den, nm[q8 * 8 + 1] * inv_den),
                                     pack_bf16(nm[q8 * 8 + 2] * inv_den, nm[q8 * 8 + 3] * inv_den),
                                     pack_bf16(nm[q8 * 8 + 4] * inv_den, nm[q8 * 8 + 5] * inv_den),
                                     pack_bf16(nm[q8 * 8 + 6] * inv_den, nm[q8 * 8 + 7] * inv_den));
          *reinterpret_cast<uint4*>(Olt + (e0 >> 6) * C::kSubS + sw128_chunk(tid, (e0 & 63) >> 3)) = v;
        }
      }
      fence_async_smem();
      tc_fence_before();
      named_bar(1, 128);
      if (tid == 0) mbar_arrive(bar(bOlFull));
      wait_w(bYFull, 0);
      tc_fence_after();
    }
#pragma unroll 1
    for (int ch = 0; ch < D / 32; ++ch) {
      float o[32], x[32];
      if (use_y) tmem_ld32(tq + C::cY + ch * 32, x);
      else if (has_marg) load_num(ch, x);
      tmem_ld32(tq + C::cO + ch * 32, o);
      tmem_wait_ld();
      float out[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float os = o[i] * inv_l;
        const float ol = use_y ? x[i] : (has_marg ? x[i] * inv_den : 0.0f);
        out[i] = MODE == kModeSLA2 ? alpha * os + (1.0f - alpha) * ol : os + ol;
      }
      if (srow) {
        save_row(a.save_os, ch, o, inv_l);
        if (!use_y && has_marg) save_row(a.save_ol, ch, x, inv_den);
        if (!has_marg) {  // no marginal block: O^l = 0 (x was never loaded)
          uint4* p = reinterpret_cast<uint4*>(a.save_ol + sidx * D + ch * 32);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) p[q8] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        const int e0 = ch * 32 + q8 * 8;
        *reinterpret_cast<uint4*>(Ot + (e0 >> 6) * C::kSubS + sw128_chunk(tid, (e0 & 63) >> 3)) =
            make_uint4(pack_bf16(out[8 * q8], out[8 * q8 + 1]), pack_bf16(out[8 * q8 + 2], out[8 * q8 + 3]),
                       pack_bf16(out[8 * q8 + 4], out[8 * q8 + 5]), pack_bf16(out[8 * q8 + 6], out[8 * q8 + 7]));
      }
    }
    fence_async_smem();
    named_bar(1, 128);
    if (tid == 0) {
      const uint32_t so = smem_u32(Ot);
#pragma unroll
      for (int s = 0; s < C::kSub; ++s) {
        tma_store_3d(&maps.o, so + s * C::kSubS, s * 64, iA * 64, bh);
        if (validB) tma_store_3d(&maps.o, so + s * C::kSubS + C::kHalf, s * 64, iB * 64, bh);
      }
      tma_store_commit_wait_read();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tb, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------
namespace {

using tc::EncodeTiledFn;
using tc::encode_fn;
using tc::map_rows;

// [D][D] bf16 (row = input dim), boxes of 64 columns x D rows.
bool map_square(CUtensorMap* m, const void* base, int D) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(D)};
  cuuint64_t strides[1] = {cuuint64_t(D) * 2};
  cuuint32_t box[2] = {64, cuuint32_t(D)};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [BH][D][D] bf16 (a matrix per head, row = input dim), boxes of 64 columns x D rows.
bool map_square_heads(CUtensorMap* m, const void* base, int D, int BH) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(D), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(D) * D * 2};
  cuuint32_t box[3] = {64, cuuint32_t(D), 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [BH][rows][D] one-byte codes viewed as 3D (D bytes, rows, BH); one box is a
// 64-row x 128-byte tile (D = 128).
bool map_codes(CUtensorMap* m, const void* base, int D, int rows, int BH) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(rows), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(D), cuuint64_t(rows) * D};
  cuuint32_t box[3] = {128, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int MODE, bool QNT = false>
cudaError_t launch_tc(const TcMaps& maps, const AttnArgs& a, int BH, cudaStream_t s) {
  const int bytes = TcCfg<D>::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D, MODE, QNT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<D, MODE, QNT><<<dim3((a.Nb + 1) / 2, BH), 192, bytes, s>>>(maps, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, int BH, int d, int mode, cudaStream_t s) {
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));
  const int Npad = a.Nb * kBlock;
  bool ok = map_rows(&maps.q, a.Q, d, a.N, Npad, BH) && map_rows(&maps.k, a.K, d, a.N, Npad, BH) &&
            map_rows(&maps.v, a.V, d, a.N, Npad, BH);
  if (ok && a.phik) ok = map_rows(&maps.phik, a.phik, d, Npad, Npad, BH);
  if (ok && a.phiq) ok = map_rows(&maps.phiq, a.phiq, d, a.N, Npad, BH);
  if (ok) ok = map_rows(&maps.o, a.O, d, a.N, Npad, BH);
  if (ok && a.w_proj) ok = map_square(&maps.w, a.w_proj, d);
  if (ok && d == 128 && mode != kModeDense)  // the d = 128 epilogue reads H_tot as a bf16 tile
    ok = a.htot16 != nullptr && map_square_heads(&maps.ht, a.htot16, d, BH);
  const bool quant = a.qcode != nullptr;
  // the quantised branch's Q tiles hold INT8 codes: its phi(Q) must come precomputed
  if (quant && a.kc + a.kn < a.Nb && a.phiq == nullptr) return cudaErrorInvalidValue;
  if (ok && quant)
    ok = d == 128 && mode != kModeDense && map_codes(&maps.qc, a.qcode, d, Npad, BH) &&
         map_codes(&maps.kc, a.kcode, d, Npad, BH) && map_codes(&maps.vc, a.vcode, d, Npad, BH);
  if (!ok) return cudaErrorInvalidValue;
  if (quant) {
    return mode == kModeSLA ? launch_tc<128, kModeSLA, true>(maps, a, BH, s)
                            : launch_tc<128, kModeSLA2, true>(maps, a, BH, s);
  }
  if (d == 128) {
    if (mode == kModeSLA) return launch_tc<128, kModeSLA>(maps, a, BH, s);
    if (mode == kModeSLA2) return launch_tc<128, kModeSLA2>(maps, a, BH, s);
    return launch_tc<128, kModeDense>(maps, a, BH, s);
  }
  if (mode == kModeSLA) return launch_tc<64, kModeSLA>(maps, a, BH, s);
  if (mode == kModeSLA2) return launch_tc<64, kModeSLA2>(maps, a, BH, s);
  return launch_tc<64, kModeDense>(maps, a, BH, s);
}

}  // namespace sla
