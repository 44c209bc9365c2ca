// backward_kernels.cuh — gradients of exact attention on sm_100a tensor cores.
//
// For O = P V with P = softmax(scale * Q Kᵀ + mask), the gradients are
//   dV = Pᵀ dO,  dP = dO Vᵀ,  dS = P * (dP - rowsum(dO * O)),
//   dQ = scale * dS K,  dK = scale * dSᵀ Q,
// with P recomputed from the log-sum-exp the forward pass saved ("Chapter 3:
// MHA Limitations, MQA, GQA, and FlashAttention", section 3.5: the saved
// log-sum-exp serves the backward pass), so no score matrix is stored.
//
// Three kernels:
//   bwd_prep_kernel     delta = rowsum(dO * O) per query row; zeroes the fp32
//                       dQ accumulator
//   bwd_main_kernel     one CTA per (batch, K/V head, 128-key block): loops
//                       over the group's query heads and the query blocks the
//                       mask allows, accumulates dK and dV of its keys in
//                       tensor memory, adds dQ contributions to the
//                       accumulator with vector atomics
//   bwd_finalize_kernel dQ accumulator -> bf16
//
// bwd_main_kernel warp roles (480 threads):
//   warps 0-7  elementwise, thread = TMEM lane = key row: P, then dS, per
//              block; at the end dK, dV. Warps w and w + 4 share the key rows
//              of lanes 32 (w % 4) .. + 31, warp w takes queries [0, 64) of a
//              block and warp w + 4 queries [64, 128), so each SM
//              sub-partition runs two of them
//   warps 8-11 dQ, thread = TMEM lane = query row: read dQ_i out of tensor
//              memory, add it to the accumulator
//   warp 12    tensor-core issuer (whole warp, one elected lane issues)
//   warp 13    TMA producer (one lane): K_j, V_j once; Q_i, dO_i per block
//              through a 2-stage ring (the next block's tiles load during this one)
//   warp 14    stages each block's lse2 / delta values in shared memory
// Per query block (tile = 128 x 128), TMEM cols [0,128) Sᵀ / Pᵀ, [128,256)
// dPᵀ / dQ_i, [256,256+D) dV, [256+D,256+2D) dK:
//   Sᵀ  = K_j Q_iᵀ        SS, both K-major (N = 128)
//   phase P: Pᵀ = exp2(Sᵀ c - lse2) as bf16 pairs, queries [0,64) over cols
//     [0,32) and queries [64,128) over cols [64,96) (each half over Sᵀ columns
//     its own warps have read); the pairs stay in registers
//   dV += Pᵀ dO_i         TS: A = Pᵀ (TMEM), B = dO_i MN-major
//   dPᵀ = V_j dO_iᵀ       SS, both K-major (N = 128)
//   phase dS: dSᵀ = Pᵀ (dPᵀ - delta) from those bf16 P, to shared memory only
//   dQ_i = dS K_j         SS: A = dS MN-major (the dSᵀ tile read transposed),
//                         B = K_j MN-major (N = D), into the dPᵀ columns
//   dK += dSᵀ Q_i         SS: A = the dSᵀ tile K-major, B = Q_i MN-major
// The next block's Sᵀ goes in as soon as dV has read Pᵀ, so the elementwise
// warps find it ready after their dS phase; the next dPᵀ follows the
// read-out of dQ_i.
// All waits are bounded (sm100_ptx.cuh).
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"

namespace attn {

// kind::f16 instruction descriptor with A MN-major too (bit 15).
__host__ __device__ constexpr uint32_t idesc_bf16_f32_amn(int M, int N, int b_mn_major) {
  return idesc_bf16_f32(M, N, b_mn_major) | (1u << 15);
}

// 32 lanes x 16 columns of 32-bit from thread i of the warp (lane base + i).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
        "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Pᵀ of one key row over 32 queries [c0, c0 + 32) of the block, as bf16 pairs:
// P = exp2(S c2 - lse2). MASK: only the queries in [c_lo, c_hi] are allowed,
// the rest get P = 0.
template <bool MASK>
__device__ __forceinline__ void bwd_p(const uint32_t* sr, const float* lsr, int c0, int c_lo, int c_hi,
                                      float c2, uint32_t* pw) {
  const float4* l4 = reinterpret_cast<const float4*>(lsr + c0);
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const float4 lv = l4[e / 4];
    const float l[4] = {lv.x, lv.y, lv.z, lv.w};
    float pp[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      pp[u] = ex2_approx(fmaf(__uint_as_float(sr[e + u]), c2, -l[u]));
      if (MASK) pp[u] = (c0 + e + u >= c_lo && c0 + e + u <= c_hi) ? pp[u] : 0.f;
    }
    pw[e / 2] = pack_bf16x2(pp[0], pp[1]);
    pw[e / 2 + 1] = pack_bf16x2(pp[2], pp[3]);
  }
}

// dSᵀ = Pᵀ (dPᵀ - delta) of one key row over 32 queries [c0, c0 + 32), from the
// bf16 pairs of Pᵀ (the values the dV product uses), as bf16 pairs.
__device__ __forceinline__ void bwd_ds(const uint32_t* dr, const uint32_t* pw, const float* dlt, int c0,
                                       uint32_t* dw) {
  const float4* d4 = reinterpret_cast<const float4*>(dlt + c0);
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const float4 dv = d4[e / 4];
    const float ds0 = bf16lo(pw[e / 2]) * (__uint_as_float(dr[e]) - dv.x);
    const float ds1 = bf16hi(pw[e / 2]) * (__uint_as_float(dr[e + 1]) - dv.y);
    const float ds2 = bf16lo(pw[e / 2 + 1]) * (__uint_as_float(dr[e + 2]) - dv.z);
    const float ds3 = bf16hi(pw[e / 2 + 1]) * (__uint_as_float(dr[e + 3]) - dv.w);
    dw[e / 2] = pack_bf16x2(ds0, ds1);
    dw[e / 2 + 1] = pack_bf16x2(ds2, ds3);
  }
}

struct BwdParams {
  const uint16_t* o;       // [B, Nq, Hq, D] bf16, forward output
  const uint16_t* dout;    // [B, Nq, Hq, D] bf16
  const float* lse;        // [B, Hq, Nq] natural log-sum-exp of the forward
  float* delta;            // [B, Hq, Nq] rowsum(dO * O)              (workspace)
  float* dq_acc;           // [B, Hq, D/4, Nq] float4, scale * dQ     (workspace)
  uint16_t* dq;            // [B, Nq, Hq, D] bf16
  uint16_t* dk;            // [B, Nk, Hkv, D] bf16
  uint16_t* dv;            // [B, Nk, Hkv, D] bf16
  int B, Hq, Hkv, Nq, Nk;
  int causal, window_left;
  float scale, scale_log2;
  int bh_chunk;            // (batch, K/V head) pairs per scheduling chunk, >= 1
};

// ---- delta = rowsum(dO * O); zero the dQ accumulator ------------------------
// One warp per (b, query row, head); lane l covers elements [l*D/32, (l+1)*D/32).
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdParams p) {
  constexpr int EPL = D / 32;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(p.B) * p.Nq * p.Hq;
  if (row >= rows) return;
  const size_t base = size_t(row) * D + lane * EPL;          // row = (b * Nq + q) * Hq + h
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; e += 2) {
    const uint32_t a = *reinterpret_cast<const uint32_t*>(p.dout + base + e);
    const uint32_t c = *reinterpret_cast<const uint32_t*>(p.o + base + e);
    acc = fmaf(bf16lo(a), bf16lo(c), acc);
    acc = fmaf(bf16hi(a), bf16hi(c), acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (in_bounds(static_cast<long long>(base) + EPL - 1, rows * D)) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) p.dq_acc[base + e] = 0.f;   // slice `row` of the buffer
  }
  if (lane == 0) {
    const int h = int(row % p.Hq);
    const long long bq = row / p.Hq;                         // b * Nq + q
    const int q = int(bq % p.Nq);
    const int b = int(bq / p.Nq);
    const size_t di = (size_t(b) * p.Hq + h) * p.Nq + q;
    if (in_bounds(static_cast<long long>(di), rows)) p.delta[di] = acc;
  }
}

// ---- dQ accumulator (already scaled) -> bf16 --------------------------------
// The accumulator keeps each 4-wide column chunk of a (batch, head) contiguous
// over the queries, so that a warp's atomics (32 consecutive queries) cover
// 512 contiguous bytes. One CTA turns 64 queries of one (batch, head) back
// into rows of dq through shared memory: reads and writes both coalesced.
constexpr int kFinQ = 64;

template <int D>
__global__ void __launch_bounds__(256) bwd_finalize_kernel(const BwdParams p) {
  constexpr int C4 = D / 4;
  __shared__ float4 tile[C4][kFinQ + 1];
  const int nqt = (p.Nq + kFinQ - 1) / kFinQ;
  const long long bh = static_cast<long long>(blockIdx.x) / nqt;      // b * Hq + hq
  const int q0 = int(static_cast<long long>(blockIdx.x) % nqt) * kFinQ;
  const float4* src = reinterpret_cast<const float4*>(p.dq_acc) + size_t(bh) * C4 * p.Nq;
  for (int idx = threadIdx.x; idx < C4 * kFinQ; idx += blockDim.x) {
    const int c = idx / kFinQ, ql = idx % kFinQ;
    const int q = q0 + ql;
    tile[c][ql] = q < p.Nq ? src[size_t(c) * p.Nq + q] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  const int hq = int(bh % p.Hq), b = int(bh / p.Hq);
  for (int idx = threadIdx.x; idx < kFinQ * (D / 8); idx += blockDim.x) {
    const int ql = idx / (D / 8), g = idx % (D / 8);
    const int q = q0 + ql;
    if (q >= p.Nq) continue;
    if (!in_bounds((static_cast<long long>(b) * p.Nq + q) * p.Hq + hq, static_cast<long long>(p.B) * p.Nq * p.Hq))
      continue;
    const float4 a = tile[2 * g][ql], c = tile[2 * g + 1][ql];
    uint4 v;
    v.x = pack_bf16x2(a.x, a.y);
    v.y = pack_bf16x2(a.z, a.w);
    v.z = pack_bf16x2(c.x, c.y);
    v.w = pack_bf16x2(c.z, c.w);
    reinterpret_cast<uint4*>(p.dq + ((size_t(b) * p.Nq + q) * p.Hq + hq) * D)[g] = v;
  }
}

template <int D>
struct BwdLayout {
  static constexpr int TILE = 128 * D * 2;                 // 128 rows x D bf16
  static constexpr int HALF = 128 * 128;                   // 128 rows x 64 columns, swizzled
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;              // Q_i, 2 stages
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;          // dO_i, 2 stages
  static constexpr int OFF_DS = OFF_DO + 2 * TILE;         // dSᵀ [128 keys][128 queries] bf16
  static constexpr int OFF_LD = OFF_DS + 2 * HALF;         // f32 lse2[128], delta[128]
  static constexpr int OFF_BAR = OFF_LD + 2 * 128 * 4;
  static constexpr int B_KV = 0;     // K_j, V_j loaded
  static constexpr int B_QD = 1;     // Q_i, dO_i loaded, + stage
  static constexpr int B_QDE = 3;    // Q_i, dO_i stage free again, + stage
  static constexpr int B_SS = 5;     // Sᵀ in TMEM
  static constexpr int B_SP = 6;     // dPᵀ in TMEM (and the previous dQ product done)
  static constexpr int B_PA = 7;     // Pᵀ written (256 elementwise arrivals)
  static constexpr int B_PB = 8;     // dSᵀ written to shared memory (256 arrivals)
  static constexpr int B_DVD = 9;    // dV product of the block complete (issuer only)
  static constexpr int B_QR = 10;    // dQ_i in TMEM
  static constexpr int B_QF = 11;    // dQ_i read out (128 dQ-warp arrivals)
  static constexpr int B_DONE = 12;  // every dK / dV product complete
  static constexpr int B_LD = 13;    // block lse2 / delta values in shared memory (32 arrivals)
  static constexpr int NBAR = 14;
  // [0] TMEM base, [1] abort flag; [2..4] query blocks the producer loaded, the
  // elementwise warps and the issuer completed (compared at the end of the CTA
  // in the bounds-checking debug build)
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 32;
  static constexpr int SMEM_ALLOC = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_ST = 0, COL_DPT = 128, COL_DV = 256, COL_DK = 256 + D;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0);
  static constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, D, 1);
  static constexpr uint32_t IDESC_DQ = idesc_bf16_f32_amn(128, D, 1);
};

constexpr int kBwdThreads = 480;

// Query blocks that hold at least one allowed (query, key) pair with a key in
// [kb0, kb1]: [i_lo, i_hi], empty when i_hi < i_lo.
__device__ __forceinline__ void bwd_qblocks(const BwdParams& p, int kb0, int kb1, int& i_lo, int& i_hi) {
  const int off = p.Nk - p.Nq;                               // qpos = q + off
  int q_lo = p.causal ? max(0, kb0 - off) : 0;
  int q_hi = p.window_left >= 0 ? min(p.Nq - 1, kb1 + p.window_left - off) : p.Nq - 1;
  if (q_hi < q_lo) { i_lo = 0; i_hi = -1; return; }
  i_lo = q_lo / 128;
  i_hi = q_hi / 128;
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::OFF_BAR + 8u * uint32_t(i); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // One CTA per (batch, K/V head, 128-key block) on a 1-D grid. The (batch,
  // head) pairs go in chunks of bh_chunk, whose Q, dO and dQ rows stay in L2
  // together; inside a chunk the key blocks run heaviest first (most query
  // blocks), so the last CTAs to start are the short ones.
  const int nkb = (p.Nk + 127) / 128, nbh = p.B * p.Hkv;
  const int per_chunk = p.bh_chunk * nkb;
  const int chunk = int(blockIdx.x) / per_chunk, r = int(blockIdx.x) % per_chunk;
  const int cs = min(p.bh_chunk, nbh - chunk * p.bh_chunk);
  const int jj = r / cs, bh = chunk * p.bh_chunk + r % cs;
  // causal: earlier key blocks see more queries; window only: later ones do
  const int j = (p.causal || p.window_left < 0) ? jj : nkb - 1 - jj;
  const int hkv = bh % p.Hkv, b = bh / p.Hkv;
  const int G = p.Hq / p.Hkv;
  const int kb0 = j * 128, kb1 = min(kb0 + 127, p.Nk - 1);
  int i_lo, i_hi;
  bwd_qblocks(p, kb0, kb1, i_lo, i_hi);
  const int nblk = i_hi - i_lo + 1;                          // per query head (<= 0: none)
  const int total = nblk > 0 ? G * nblk : 0;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::B_KV), 1);
    for (int st = 0; st < 2; ++st) {
      mbar_init(bar(L::B_QD + st), 1);
      mbar_init(bar(L::B_QDE + st), 1);
    }
    mbar_init(bar(L::B_SS), 1);
    mbar_init(bar(L::B_SP), 1);
    mbar_init(bar(L::B_PA), 256);
    mbar_init(bar(L::B_PB), 256);
    mbar_init(bar(L::B_DVD), 1);
    mbar_init(bar(L::B_QR), 1);
    mbar_init(bar(L::B_QF), 128);
    mbar_init(bar(L::B_DONE), 1);
    mbar_init(bar(L::B_LD), 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(smem_u32(tmem_holder), L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp < 8) {
    // ======================= elementwise warps ==============================
    // warps w and w + 4 share TMEM lanes 32 (w % 4) .. + 31 (their key rows);
    // warp w takes queries [0, 64) of each block, warp w + 4 queries [64, 128)
    const int t = int(threadIdx.x) & 127;                    // TMEM lane
    const int hh = warp >> 2;                                // query half
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tST = tmem + lane_off + L::COL_ST, tDPT = tmem + lane_off + L::COL_DPT;
    const float* lsr = reinterpret_cast<const float*>(smem + L::OFF_LD);   // lse2[128]
    const float* dlt = lsr + 128;                                           // delta[128]
    const int key = kb0 + t;
    const int off = p.Nk - p.Nq;
    const float c2 = p.scale_log2;
    bool ok = true;
    for (int n = 0; ok && n < total; ++n) {
      const int i = i_lo + n % nblk;
      const uint32_t par = uint32_t(n & 1);
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_SS), par, abort_flag)))) break;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_LD), par, abort_flag)))) break;
      tc_fence_after();
      // allowed queries of this key within the block: [c_lo, c_hi]
      const int q0 = i * 128;
      int c_lo = 0, c_hi = min(127, p.Nq - 1 - q0);
      if (key >= p.Nk) c_hi = -1;
      if (p.causal) c_lo = max(c_lo, key - off - q0);                    // key <= q + off
      if (p.window_left >= 0) c_hi = min(c_hi, key + p.window_left - off - q0);
      // phase A, 32 queries at a time: Pᵀ over columns of Sᵀ this warp has
      // already read (queries [64h + 32c, +32) -> columns [64h + 16c, +16)); the
      // bf16 pairs stay in registers
      uint32_t pw[2][16];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c0 = 64 * hh + 32 * cc;
        uint32_t sr[32];
        tmem_ld32(tST + c0, sr);
        tmem_wait_ld();
        if (__all_sync(0xffffffffu, c_lo <= c0 && c_hi >= c0 + 31))
          bwd_p<false>(sr, lsr, c0, c_lo, c_hi, c2, pw[cc]);
        else
          bwd_p<true>(sr, lsr, c0, c_lo, c_hi, c2, pw[cc]);
        tmem_st16(tST + 64 * hh + 16 * cc, pw[cc]);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::B_PA));
      // phase B: dSᵀ once dPᵀ is in TMEM. B_SP also covers the previous dQ
      // product, the last reader of the dS tile in shared memory.
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_SP), par, abort_flag)))) break;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c0 = 64 * hh + 32 * cc;
        uint32_t dr[32], dw[16];
        tmem_ld32(tDPT + c0, dr);
        tmem_wait_ld();
        bwd_ds(dr, pw[cc], dlt, c0, dw);
        // dSᵀ row of this key -> shared memory block hh (queries 64hh..64hh+63),
        // 16-byte chunks swizzled by (row & 7)
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int chunk = 4 * cc + ch;
          const uint32_t addr = sb + L::OFF_DS + hh * L::HALF + t * 128 + ((chunk ^ (t & 7)) * 16);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                       ::"r"(addr), "r"(dw[4 * ch]), "r"(dw[4 * ch + 1]), "r"(dw[4 * ch + 2]),
                       "r"(dw[4 * ch + 3]) : "memory");
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(bar(L::B_PB));
      if (threadIdx.x == 0) reinterpret_cast<volatile int*>(smem + L::OFF_MISC)[3] = n + 1;
    }
    // ---- dK, dV of this key row ---------------------------------------------
    const bool have = ok && total > 0 &&
                      __all_sync(0xffffffffu, mbar_wait(bar(L::B_DONE), 0u, abort_flag));
    if (have) tc_fence_after();
    // Each warp stages its 32 key rows of dV, then dK (scaled), for its
    // 64-column half hh, as 4 KB blocks of 32 rows x 64 columns in the 128-byte
    // swizzled layout of the tensor maps, in the Q ring (free once every product
    // has completed); lane 0 stores the blocks. Rows past Nk fall outside the
    // maps and are not written. At D = 64 the warps of half 0 do it all.
    constexpr int NH = D / 64;
    const int wk0 = kb0 + 32 * (warp & 3);
    if ((have || (ok && total == 0)) && wk0 < p.Nk && hh < NH) {
      const uint32_t stg = sb + L::OFF_Q + uint32_t(warp & 3) * (2 * NH * 4096);
#pragma unroll
      for (int m = 0; m < 2; ++m) {                          // 0: dV, 1: dK (scaled)
        const float f = m ? p.scale : 1.f;
#pragma unroll
        for (int c = 2 * hh; c < 2 * hh + 2; ++c) {
          uint32_t r[32];
          if (have) {
            tmem_ld32(tmem + lane_off + (m ? L::COL_DK : L::COL_DV) + 32 * c, r);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = 0u;
          }
          const uint32_t blk = stg + uint32_t(m * NH + c / 2) * 4096u + uint32_t(lane) * 128u;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            st_shared_v4(blk + uint32_t(((4 * (c & 1) + e) ^ (lane & 7)) << 4),
                         pack_bf16x2(__uint_as_float(r[8 * e]) * f, __uint_as_float(r[8 * e + 1]) * f),
                         pack_bf16x2(__uint_as_float(r[8 * e + 2]) * f, __uint_as_float(r[8 * e + 3]) * f),
                         pack_bf16x2(__uint_as_float(r[8 * e + 4]) * f, __uint_as_float(r[8 * e + 5]) * f),
                         pack_bf16x2(__uint_as_float(r[8 * e + 6]) * f, __uint_as_float(r[8 * e + 7]) * f));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && in_bounds(b, p.B) && in_bounds(hkv, p.Hkv)) {
#pragma unroll
        for (int m = 0; m < 2; ++m)
          tma_store_4d(m ? &tmDK : &tmDV, stg + uint32_t(m * NH + hh) * 4096u, 64 * hh, hkv, wk0, b);
        bulk_commit_group();
        bulk_wait_all();                    // shared memory outlives the stores
      }
    }
  } else if (warp < 12) {
    // ======================= dQ warps ========================================
    const int r = int(threadIdx.x) - 256;                    // TMEM lane = query row in the block
    const uint32_t tDQ = tmem + (uint32_t((warp - 8) * 32) << 16) + L::COL_DPT;
    for (int n = 0; n < total; ++n) {
      const int hq = hkv * G + n / nblk, q = (i_lo + n % nblk) * 128 + r;
      const uint32_t par = uint32_t(n & 1);
      if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_QR), par, abort_flag))) break;
      tc_fence_after();
      const bool qok = q < p.Nq && in_bounds((static_cast<long long>(b) * p.Hq + hq) * p.Nq + q,
                                             static_cast<long long>(p.B) * p.Hq * p.Nq);
      // chunk e of query q: the warp's 32 queries are 32 adjacent float4
      float4* dst = reinterpret_cast<float4*>(p.dq_acc) + (size_t(b) * p.Hq + hq) * (D / 4) * p.Nq +
                    (qok ? q : 0);
      // 64 columns at a time (the register budget of 15 warps); the columns
      // are released once the last ones are read
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf) {
        uint32_t qr[64];
        tmem_ld32(tDQ + 64 * hf, qr);
        tmem_ld32(tDQ + 64 * hf + 32, qr + 32);
        tmem_wait_ld();
        if (hf == D / 64 - 1) {
          tc_fence_before();
          mbar_arrive(bar(L::B_QF));
        }
        if (qok) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            atomicAdd(dst + size_t(16 * hf + e) * p.Nq,
                      make_float4(__uint_as_float(qr[4 * e]) * p.scale, __uint_as_float(qr[4 * e + 1]) * p.scale,
                                  __uint_as_float(qr[4 * e + 2]) * p.scale, __uint_as_float(qr[4 * e + 3]) * p.scale));
        }
      }
    }
  } else if (warp == 12) {
    // ======================= tensor-core issuer ==============================
    auto wwait = [&](int bi, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar(bi), parity, abort_flag));
    };
    auto commit = [&](int bi) { if (elect_one()) tc_commit(bar(bi)); };
    // K-major views (Sᵀ, dPᵀ) and MN-major views (dK, dV, dQ) of the same tiles
    const uint64_t dK_k = smem_desc_sw128(sb + L::OFF_K, 16, 1024);
    const uint64_t dV_k = smem_desc_sw128(sb + L::OFF_V, 16, 1024);
    const uint64_t dQ_k = smem_desc_sw128(sb + L::OFF_Q, 16, 1024);
    const uint64_t dO_k = smem_desc_sw128(sb + L::OFF_DO, 16, 1024);
    const uint64_t dQ_mn = smem_desc_sw128(sb + L::OFF_Q, L::HALF, 1024);
    const uint64_t dO_mn = smem_desc_sw128(sb + L::OFF_DO, L::HALF, 1024);
    const uint64_t dS_mn = smem_desc_sw128(sb + L::OFF_DS, L::HALF, 1024);
    const uint64_t dS_k = smem_desc_sw128(sb + L::OFF_DS, 16, 1024);
    const uint64_t dKj_mn = smem_desc_sw128(sb + L::OFF_K, L::HALF, 1024);
    const uint32_t tST = tmem + L::COL_ST, tDPT = tmem + L::COL_DPT;
    const uint32_t tDV = tmem + L::COL_DV, tDK = tmem + L::COL_DK;
    // A_j X_iᵀ (K = d) into TMEM cols [col, col + 128): Sᵀ (A = K, X = Q) or
    // dPᵀ (A = V, X = dO) of block n
    auto issue_rows = [&](uint32_t dst, uint64_t a_k, uint64_t x_k, int n) {
      const uint32_t so = uint32_t(((n & 1) * L::TILE) >> 4);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t o = ((k / 4) * L::HALF + (k % 4) * 32) >> 4;
        if (elect_one()) mma_ss(dst, a_k + o, x_k + so + o, L::IDESC_S, k > 0 ? 1u : 0u);
      }
    };
    bool alive = total > 0 && wwait(L::B_KV, 0u) && wwait(L::B_QD, 0u);
    if (alive) {
      tc_fence_after();
      issue_rows(tST, dK_k, dQ_k, 0);
      commit(L::B_SS);
    }
    for (int n = 0; alive && n < total; ++n) {
      const uint32_t par = uint32_t(n & 1);
      const int stg = n & 1;                                     // Q/dO stage of this block
      const uint32_t so = uint32_t(stg * (L::TILE >> 4));       // its descriptor offset
      const bool next = n + 1 < total;
      // dPᵀ once dQ of the previous block (cols [128, 128 + D)) is read out;
      // the commit also covers that dQ product, the last reader of the dS tile
      if (n > 0 && !(alive = wwait(L::B_QF, par ^ 1u))) break;
      tc_fence_after();
      issue_rows(tDPT, dV_k, dO_k, n);
      commit(L::B_SP);
      // dV += Pᵀ dO_i (K = 128 queries, 16 per MMA) once Pᵀ is in TMEM
      if (!(alive = wwait(L::B_PA, par))) break;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t o = (k * 16 * 128) >> 4;
        // Pᵀ of queries [16k, 16k + 16): columns 8k.. for the first half, 32 + 8k..
        // for the second (written over the Sᵀ columns that half's warps read)
        const uint32_t pa = uint32_t(8 * k + (k >= 4 ? 32 : 0));
        if (elect_one()) mma_ts(tDV, tST + pa, dO_mn + so + o, L::IDESC_KV, (n > 0 || k > 0) ? 1u : 0u);
      }
      if (next) {
        // Sᵀ of the next block over cols [0, 128): Pᵀ (cols [0, 64)) must have
        // been read by the dV product, and the elementwise warps are done with Sᵀ
        commit(L::B_DVD);
        if (!(alive = wwait(L::B_QD + ((n + 1) & 1), uint32_t(((n + 1) >> 1) & 1)))) break;
        if (!(alive = wwait(L::B_DVD, par))) break;
        tc_fence_after();
        issue_rows(tST, dK_k, dQ_k, n + 1);
        commit(L::B_SS);
      }
      // once dSᵀ is in shared memory: dQ_i = dS K_j (K = 128 keys) into the dPᵀ
      // columns, already read, then dK += dSᵀ Q_i with dSᵀ read K-major from the
      // same tile (K = 128 queries, 16 per MMA)
      if (!(alive = wwait(L::B_PB, par))) break;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t o = (k * 16 * 128) >> 4;
        if (elect_one()) mma_ss(tDPT, dS_mn + o, dKj_mn + o, L::IDESC_DQ, k > 0 ? 1u : 0u);
      }
      commit(L::B_QR);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t oa = ((k / 4) * L::HALF + (k % 4) * 32) >> 4;
        const uint32_t ob = (k * 16 * 128) >> 4;
        if (elect_one()) mma_ss(tDK, dS_k + oa, dQ_mn + so + ob, L::IDESC_KV, (n > 0 || k > 0) ? 1u : 0u);
      }
      commit(L::B_QDE + stg);                   // dK is the last reader of Q_i, dO_i
      if (lane == 0) reinterpret_cast<volatile int*>(smem + L::OFF_MISC)[4] = n + 1;
    }
    if (total > 0) {
      commit(L::B_DONE);                        // also drains every issued product
      mbar_wait(bar(L::B_DONE), 0, nullptr);
    }
    __syncwarp();
  } else if (warp == 13) {
    // ======================= TMA producer ====================================
    if (lane == 0 && total > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(bar(L::B_KV), 2 * L::TILE);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_4d(sb + L::OFF_K + c * L::HALF, &tmK, bar(L::B_KV), c * 64, hkv, kb0, b);
        tma_load_4d(sb + L::OFF_V + c * L::HALF, &tmV, bar(L::B_KV), c * 64, hkv, kb0, b);
      }
      int issued = 0;
      for (int n = 0; n < total; ++n) {
        const int g = n / nblk, i = i_lo + n % nblk;
        const int hq = hkv * G + g;
        const int stg = n & 1;
        // the stage is free once the products of block n - 2 completed
        if (n >= 2 && !mbar_wait(bar(L::B_QDE + stg), uint32_t(((n >> 1) - 1) & 1), abort_flag)) break;
        mbar_arrive_expect_tx(bar(L::B_QD + stg), 2 * L::TILE);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_4d(sb + L::OFF_Q + stg * L::TILE + c * L::HALF, &tmQ, bar(L::B_QD + stg), c * 64,
                      hq, i * 128, b);
          tma_load_4d(sb + L::OFF_DO + stg * L::TILE + c * L::HALF, &tmDO, bar(L::B_QD + stg),
                      c * 64, hq, i * 128, b);
        }
        issued = n + 1;
      }
      reinterpret_cast<volatile int*>(smem + L::OFF_MISC)[2] = issued;
      // no copy may still be landing at exit
      mbar_wait(bar(L::B_KV), 0, nullptr);
      for (int n = max(0, issued - 2); n < issued; ++n)
        mbar_wait(bar(L::B_QD + (n & 1)), uint32_t((n >> 1) & 1), nullptr);
    }
    __syncwarp();
  }

  if (warp == 14) {
    // ======================= lse / delta stager ==============================
    // lane l stages query rows l, l + 32, l + 64, l + 96 of each block once
    // every elementwise thread arrived on B_PB of the block before (its last
    // read of those values); the loads go out before that wait
    float* lse2_s = reinterpret_cast<float*>(smem + L::OFF_LD);
    float* delta_s = lse2_s + 128;
    for (int n = 0; n < total; ++n) {
      const int hq = hkv * G + n / nblk, qb = (i_lo + n % nblk) * 128;
      float l2[4], dl[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int q = qb + lane + 32 * u;
        const bool qv = q < p.Nq;
        const float l = qv ? __ldg(p.lse + (size_t(b) * p.Hq + hq) * p.Nq + q) : 0.f;
        l2[u] = (qv && l > -CUDART_INF_F) ? l * 1.4426950408889634f : 0.f;
        dl[u] = qv ? __ldg(p.delta + (size_t(b) * p.Hq + hq) * p.Nq + q) : 0.f;
      }
      if (n > 0 && !__all_sync(0xffffffffu, mbar_wait(bar(L::B_PB), uint32_t((n - 1) & 1), abort_flag)))
        break;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        lse2_s[lane + 32 * u] = l2[u];
        delta_s[lane + 32 * u] = dl[u];
      }
      mbar_arrive(bar(L::B_LD));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (kDebugBounds && threadIdx.x == 0 && *abort_flag == 0 && total > 0) {
    // every role went through all the CTA's query blocks
    const volatile int* cnt = reinterpret_cast<const volatile int*>(smem + L::OFF_MISC);
    (void)(same_count(cnt[2], total) && same_count(cnt[3], total) && same_count(cnt[4], total));
  }
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace attn
