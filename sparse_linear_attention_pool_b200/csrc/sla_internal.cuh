// Internal declarations shared by the library's translation units: the
// workspace layout, launcher prototypes and small device helpers.
#pragma once

#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sla.h"

namespace sla {

constexpr int kBlock = SLA_BLOCK;  // bq = bkv = 64 tokens

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Status-word codes written by kernels into the first bytes of the workspace.
enum DeviceStatus : int { kDevOk = 0, kDevTimeout = 1, kDevBadIndex = 2 };

// Device address of sla_forward_noalloc's static workspace on the current
// device (looked up once per device; defined in noalloc.cu).
sla_status noalloc_workspace_address(void** out);

// Tokens per CTA in the phi(K) / h / z pass of the general path (8 blocks).
constexpr int kHzChunk = 512;
// The streaming passes (bf16, d = 128) split each head into chunks of
// consecutive blocks so that the grid is about this many CTAs: two per SM of
// a 148-SM B200, one wave.
constexpr int kStreamCtas = 296;

// Derived sizes and the byte offsets of every workspace region.
struct Layout {
  int B, H, BH, N, Npad, Nb, d, kc, kn;
  int nchunk;     // chunks per head of the phi(K) / h / z pass (one partial H, Z each)
  int stream_cb;  // blocks per chunk
  bool stream;    // bf16 at d = 128: q_stream / kv_stream kernels (pool, phi and
                  // the partial sums in two passes over Q and K, V)
  bool quant;  // INT8 / FP8 sparse branch: regions qcode .. vscale are present
  bool linear;  // a marginal block exists (the linear branch is computed)
  bool pre;     // phi(Q) and Z_i are precomputed (regions phiq, zi) instead of
                // formed inside the attention kernel
  size_t status, qbar, kbar, scores, mc, crit, neg, phik, zblk, hpart, zpart, htot32, htot16, ztot, phiq, zi;
  size_t qcode, kcode, vcode, qscale, kscale, vscale, total;
};

inline Layout make_layout(const sla_params& p) {
  Layout L{};
  L.B = p.B;
  L.H = p.H;
  L.BH = p.B * p.H;
  L.N = p.N;
  L.Nb = (p.N + kBlock - 1) / kBlock;
  L.Npad = L.Nb * kBlock;
  L.d = p.d;
  L.kc = p.k_crit;
  L.kn = p.k_neg;
  L.quant = p.precision == SLA_PREC_I8QK_F8PV;
  L.stream = p.d == 128 && !L.quant;
  if (L.stream) {
    const int per_head = std::max(1, std::min(L.Nb, kStreamCtas / std::max(1, L.BH)));
    L.stream_cb = (L.Nb + per_head - 1) / per_head;
  } else {
    L.stream_cb = kHzChunk / kBlock;
  }
  L.nchunk = (L.Nb + L.stream_cb - 1) / L.stream_cb;
  const size_t BH = size_t(L.BH), Nb = size_t(L.Nb), d = size_t(L.d);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.status = take(256);
  L.qbar = take(BH * Nb * d * 4);
  L.kbar = take(BH * Nb * d * 4);
  L.scores = take(BH * Nb * Nb * 4);
  L.mc = take(BH * Nb * Nb);
  L.crit = take(BH * Nb * size_t(L.kc) * 4);
  L.neg = take(BH * Nb * size_t(L.kn > 0 ? L.kn : 1) * 4);
  L.phik = take(BH * size_t(L.Npad) * d * 2);
  L.zblk = take(BH * Nb * d * 4);
  L.hpart = take(BH * size_t(L.nchunk) * d * d * 4);
  L.zpart = take(BH * size_t(L.nchunk) * d * 4);
  L.htot32 = take(BH * d * d * 4);
  L.htot16 = take(BH * d * d * 2);
  L.ztot = take(BH * d * 4);
  L.linear = L.kc + L.kn < L.Nb;
  // The attention kernel forms Z_i (about 350 cycles per excluded block) and
  // phi(Q) (about 8000 cycles) itself while the excluded-block products of
  // phase 2 stream (about 1260 cycles per negligible block at d = 128); when
  // phase 2 is too short to hide that, both are precomputed instead. The
  // quantised branch always precomputes: its Q tiles hold INT8 codes.
  L.pre = L.linear && (p.precision == SLA_PREC_I8QK_F8PV ||
                       size_t(L.kn) * 1260 < size_t(L.kc + L.kn) * 350 + 8000);
  L.phiq = take(L.pre ? BH * size_t(L.Npad) * d * 2 : 0);  // phi(Q) bf16 [BH, Npad, d]
  L.zi = take(L.pre ? BH * Nb * d * 4 : 0);               // Z_i fp32 [BH, Nb, d]
  const size_t codes = L.quant ? BH * size_t(L.Npad) * d : 0;
  const size_t scales = L.quant ? BH * Nb * 4 : 0;
  L.qcode = take(codes);  // int8 [BH, Npad, d]
  L.kcode = take(codes);  // int8 [BH, Npad, d]
  L.vcode = take(codes);  // e4m3 [BH, Npad, d]
  L.qscale = take(scales);
  L.kscale = take(scales);
  L.vscale = take(scales);
  L.total = off;
  return L;
}

// ---- launchers (each enqueues on `s`; returns cudaGetLastError()) ----
cudaError_t launch_pool(const Layout& L, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                        const __nv_bfloat16* proj_q, const __nv_bfloat16* proj_k, float* qbar,
                        float* kbar, int8_t* qcode, int8_t* kcode, float* qscale, float* kscale,
                        __nv_bfloat16* phiq, int phi_elu1, cudaStream_t s);
cudaError_t launch_scores(const Layout& L, const float* qbar, const float* kbar, float* scores,
                          cudaStream_t s);
// streaming passes (L.stream): Q side (qbar, phi(Q) when phiq != null) and
// K / V side (kbar, phi(K), z_j, the chunks' partial H and Z)
cudaError_t launch_q_stream(const Layout& L, const __nv_bfloat16* Q, const __nv_bfloat16* proj_q, float* qbar,
                            __nv_bfloat16* phiq, int phi_elu1, int* status, cudaStream_t s);
cudaError_t launch_kv_stream(const Layout& L, const __nv_bfloat16* K, const __nv_bfloat16* V,
                             const __nv_bfloat16* proj_k, float* kbar, __nv_bfloat16* phik, float* zblk,
                             float* hpart, float* zpart, int phi_elu1, int* status, cudaStream_t s);
cudaError_t launch_classify(const Layout& L, const float* scores, int8_t* mc, int32_t* crit,
                            int32_t* neg, cudaStream_t s);
cudaError_t launch_phik_hz(const Layout& L, const __nv_bfloat16* K, const __nv_bfloat16* V,
                           __nv_bfloat16* phik, float* zblk, float* hpart, float* zpart,
                           uint8_t* vcode, float* vscale, int phi_elu1, cudaStream_t s);
cudaError_t launch_hz_reduce(const Layout& L, const float* zpart, const float* hpart, float* htot32, __nv_bfloat16* htot16,
                             float* ztot, cudaStream_t s);
// Z_i = Z_tot - sum of z_j over the excluded blocks of query block i
cudaError_t launch_zi(const Layout& L, const int32_t* crit, const int32_t* neg, const float* zblk,
                      const float* ztot, float* zi, int* status, cudaStream_t s);
// SoftTop-k of Pc = softmax(scale s) per row: m, lambda (may be null), pc (may be null)
cudaError_t launch_soft_topk(const Layout& L, const float* scores, float* m, float* lambda, float* pc,
                             float scale, float tau, cudaStream_t s);

struct AttnArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  __nv_bfloat16* O;
  const __nv_bfloat16* phik;   // [BH, Npad, d]
  const int32_t* crit;         // [BH, Nb, kc]
  const int32_t* neg;          // [BH, Nb, kn]
  const float* htot32;         // [BH, d, d]  H_tot = sum_j phi(K_j)^T V_j
  const __nv_bfloat16* htot16; // [BH, d, d]  H_tot rounded to bf16 (read at d = 128)
  const __nv_bfloat16* phiq;   // [BH, Npad, d] phi(Q), or null: formed in the kernel
  const float* zi;             // [BH, Nb, d] Z_i, or null: formed in the kernel
  const float* ztot;           // [BH, d] Z_tot (in-kernel Z_i)
  const float* zblk;           // [BH, Nb, d] z_j (in-kernel Z_i)
  int phi_elu1;                // phi = elu + 1 elementwise (else softmax over d)
  const __nv_bfloat16* w_proj; // [d, d] or null
  const float* alpha;          // [H] or null
  int* status;                 // device status word (null: not reported)
  // quantised sparse branch (null when the precision is bf16)
  const int8_t* qcode;         // [BH, Npad, d] int8
  const int8_t* kcode;         // [BH, Npad, d] int8
  const uint8_t* vcode;        // [BH, Npad, d] e4m3
  const float* qscale;         // [BH, Nb]
  const float* kscale;         // [BH, Nb]
  const float* vscale;         // [BH, Nb]
  int H, N, Nb, kc, kn;
  float scale_log2;            // softmax scale * log2(e)
  // training forward (bf16 only; null otherwise): what the backward reads
  __nv_bfloat16* save_os;      // [BH, Npad, d] O^s
  __nv_bfloat16* save_ol;      // [BH, Npad, d] O^l (before SLA's W)
  float* save_lse;             // [BH, Npad] log sum exp(scale q.k) over the critical keys
  float* save_den;             // [BH, Npad] phi(q) . Z_i (0 without a marginal block)
};
enum AttnMode { kModeSLA = 0, kModeSLA2 = 1, kModeDense = 2 };
cudaError_t launch_attention(const AttnArgs& a, int BH, int d, int mode, cudaStream_t s);

// Backward workspace: per-row and per-block intermediates of the gradient.
struct BwLayout {
  int B, H, BH, N, Npad, Nb, d, kc, kn;
  bool linear, sla;
  size_t dnum, phiq, drow, dden, dzblk, dztot, hblk, dhblk, dhtot, dwpart, dapart, colc, cole, cntc, cnte, dks, dvs, dqs, total;
};

inline BwLayout make_bw_layout(const sla_params& p) {
  BwLayout L{};
  L.B = p.B;
  L.H = p.H;
  L.BH = p.B * p.H;
  L.N = p.N;
  L.Nb = (p.N + kBlock - 1) / kBlock;
  L.Npad = L.Nb * kBlock;
  L.d = p.d;
  L.kc = p.k_crit;
  L.kn = p.k_neg;
  L.linear = L.kc + L.kn < L.Nb;
  L.sla = p.variant == SLA_VARIANT_SLA;
  const size_t BH = size_t(L.BH), Nb = size_t(L.Nb), d = size_t(L.d), rows = BH * size_t(L.Npad);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.dnum = take(rows * d * 2);               // bf16 dO^l / den
  L.phiq = take(rows * d * 2);               // bf16 phi(Q)
  L.drow = take(rows * 4);                   // dO^s . O^s
  L.dden = take(rows * 4);                   // -(dO^l . O^l) / den
  L.dzblk = take(BH * Nb * d * 4);           // dZ_i
  L.dztot = take(BH * d * 4);
  L.hblk = take(L.linear ? BH * Nb * d * d * 2 : 0);   // h_j, bf16
  L.dhblk = take(L.linear ? BH * Nb * d * d * 2 : 0);  // dH_i, bf16
  L.dhtot = take(BH * d * d * 4);
  L.dwpart = take(L.sla ? BH * Nb * d * d * 4 : 0);    // per-block O^l^T dO
  L.dapart = take(BH * Nb * 4);                        // per-block dO . (O^s - O^l), [H][B][Nb]
  L.colc = take(BH * Nb * Nb * 4);
  L.cole = take(BH * Nb * Nb * 4);
  L.cntc = take(BH * Nb * 4);
  L.cnte = take(BH * Nb * 4);
  L.dks = take(d == 128 ? rows * d * 4 : 0);  // tcgen05 sparse partials (d = 128)
  L.dvs = take(d == 128 ? rows * d * 4 : 0);
  L.dqs = take(d == 128 ? rows * d * 4 : 0);
  L.total = off;
  return L;
}

struct BwdArgs {
  BwLayout L;
  const __nv_bfloat16 *Q, *K, *V, *dO, *save_os, *save_ol, *w_proj, *phik;
  const float *save_lse, *save_den, *alpha, *htot, *ztot, *zblk;
  const int8_t* mc;
  const int32_t *crit, *neg;
  __nv_bfloat16 *dnum, *phiq;
  float *Drow, *dden, *dzblk, *dztot, *dhtot, *dwpart, *dapart;
  __nv_bfloat16 *hblk, *dhblk;  // per-block d x d, read only by the complement sums
  int *colC, *colE, *cntC, *cntE;
  float *dks, *dvs, *dqs;
  int* status;
  __nv_bfloat16 *dQ, *dK, *dV;
  float *dW, *dalpha;
  float scale;
  bool sla;
  int phi_elu1;
};
cudaError_t launch_backward(const BwdArgs& a, cudaStream_t s);

// tcgen05 sparse loop of dK / dV (d = 128): fp32 partials, dK x scale, dV x asc
struct KvTcArgs {
  const int* colC;   // [BH][Nb][Nb]
  const int* cntC;   // [BH][Nb]
  const float* lse;  // [BH][Npad], natural log
  const float* Drow; // [BH][Npad]
  const float* alpha;
  float* dKs;        // [BH][Npad][128]
  float* dVs;
  int* status;
  int H, N, Npad, Nb;
  float scale, scale_log2;
};
// tcgen05 sparse loop of dQ (d = 128): fp32 partial, x scale
struct QTcArgs {
  const int32_t* crit;  // [BH][Nb][kc]
  const float* lse;     // [BH][Npad]
  const float* Drow;    // [BH][Npad]
  const float* alpha;
  float* dQs;           // [BH][Npad][128]
  int* status;
  int H, N, Npad, Nb, kc;
  float scale, scale_log2;
};
cudaError_t launch_bwd_q_tc(const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                            const __nv_bfloat16* dO, const QTcArgs& a, int BH, cudaStream_t s);
cudaError_t launch_bwd_kv_tc(const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                             const __nv_bfloat16* dO, const KvTcArgs& a, int BH, cudaStream_t s);

// ---- device helpers ----
__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Offset (in elements) of element (row, col) of a bf16 tile with `cols`
// columns stored with a 16-byte-chunk XOR swizzle (chunk ^= row & 7): makes
// 8-row ldmatrix reads and 16-byte cp.async writes bank-conflict free.
__device__ __forceinline__ int swz(int row, int col, int cols) {
  return row * cols + ((((col >> 3) ^ (row & 7))) << 3) + (col & 7);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  int n = valid ? 16 : 0;  // n = 0 writes 16 zero bytes and reads nothing
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int n>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(n));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two floats -> packed bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Two floats -> packed FP8 e4m3 pair in the low 16 bits (lo in the low byte),
// round to nearest even, saturating to +-448.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;\n" : "=h"(r) : "f"(hi), "f"(lo));
  return uint32_t(r);
}
constexpr float kLog2e = 1.4426950408889634f;
// 2^x on the MUFU unit (approximate, flushes subnormals)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

}  // namespace sla
