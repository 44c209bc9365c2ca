// prefill_kernel.cuh — exact attention forward pass on sm_100a tensor cores.
//
// The tiled loop of "Attention Is O(n²): FlashAttention vs Linear Attention",
// section "FlashAttention — Same FLOPs, Linear Memory": for each query block,
// walk the key/value blocks, keep a running row maximum and running sum, rescale
// the accumulator when the maximum moves, divide by the sum at the end. The
// score tile never leaves the SM: it lives in tensor memory (TMEM).
//
// The kernel is persistent: one CTA (384 threads) per SM walks a static list
// of work items (longest causal rows first, boustrophedon over the CTAs). The
// K/V ring, the barrier phases and the Q buffers carry over from item to item,
// so the next item's loads and first Q.K^T overlap the current item's tail
// and epilogue. A work item is two 128-row query tiles that share every K/V
// tile:
//   * two heads of one K/V group at the same rows when Hq / Hkv is even
//     (the grouped-query map of "Chapter 3: MHA Limitations, MQA, GQA, and
//     FlashAttention", section 3.3, so each K/V tile is loaded once for both),
//   * otherwise two consecutive row blocks of one head.
// Warp roles:
//   warps 0-3  softmax for tile 0 (thread = query row = TMEM lane)
//   warps 4-7  softmax for tile 1
//   warp 8     tensor-core issuer (one lane): S_t = Q_t K_jᵀ and O_t += P_t V_j
//   warp 9     TMA producer (one lane): Q once, then K_j / V_j through a ring
//   warps 10-11 idle (register budget only)
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 after it.
// P_t is written as bf16 pairs over the first 64 columns of S_t and read by
// the P·V product straight from TMEM. At the end of an item the softmax warps
// store LSE, read O out of TMEM and write O / l: bf16 O through per-warp
// shared-memory blocks and bulk tensor stores (in the packed kernel from the
// warps whose rows all lie inside their sequence), the rest row by row from
// registers.
//
// Masks ("Modern Attention ...", section 4 for the window; bottom-right causal
// alignment): key blocks wholly outside a tile's allowed range are skipped;
// in boundary blocks the softmax warps compare element by element in the
// 32-key chunks that some row of the warp may not see in full.
// Every mbarrier wait is bounded (sm100_ptx.cuh); on a timeout the CTA stops
// issuing work, drains what it issued, frees TMEM and exits.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "sm100_ptx.cuh"

namespace attn {

// Packed-sequence schedule tables in shared memory (ints): perm[kVlMaxSeqs]
// (sequences sorted by row units, longest first), lvl[kVlMaxUnits + 1] (first
// item of unit level u), cnt[kVlMaxUnits + 1] (cnt[u]: sequences with more
// than u units), cur[kVlMaxUnits + 1] (scatter cursors). cnt and cur serve
// only the build at kernel start; their space then holds O staging blocks.
constexpr int kVlMaxSeqs = 2048;
constexpr int kVlMaxUnits = 1024;
constexpr int kVlLvl = kVlMaxSeqs;
constexpr int kVlCnt = kVlLvl + kVlMaxUnits + 1;
constexpr int kVlCur = kVlCnt + kVlMaxUnits + 1;
constexpr int kVlInts = kVlCur + kVlMaxUnits + 1;

#ifndef ATTN_VSTAGES
#define ATTN_VSTAGES 2
#endif

// Shared-memory layout. The packed-sequence kernel (VARLEN) also holds its
// schedule tables, which leave room for two V stages only at D = 128; the
// equal-length kernel has a third V stage instead (V is read by the P.V
// products, the last in a block's issue order, so its loads have the least
// lead time).
template <int D, bool VARLEN = false>
struct FwdLayout {
  static constexpr int BM = 128;                       // query rows per tile
  static constexpr int BN = 128;                       // keys per K/V tile
  static constexpr int TILE = BM * D * 2;              // bytes of a 128 x D bf16 tile
  static constexpr int HALF = 128 * 128;               // one 128-row x 64-col swizzle block
  static constexpr int STAGES = (D == 128) ? 2 : 4;    // K ring depth
  static constexpr int VSTAGES = (D == 128 && !VARLEN) ? ATTN_VSTAGES : STAGES;   // V ring depth
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * TILE;
  static constexpr int OFF_V = OFF_K + STAGES * TILE;
  // equal-length kernel: a 32-row x 64-column O staging block per softmax warp
  // for the bulk tensor stores of the epilogue (the packed kernel stores O
  // directly)
  static constexpr int OFF_OST = OFF_V + VSTAGES * TILE;
  static constexpr int OFF_BAR = OFF_OST + (VARLEN ? 0 : 2 * HALF);
  // barrier indices
  static constexpr int B_Q = 0;                         // Q tiles loaded
  static constexpr int B_QE = 1;                        // Q tiles free (all Q.K^T done)
  static constexpr int B_KF = 2;                        // + stage
  static constexpr int B_KE = B_KF + STAGES;
  static constexpr int B_VF = B_KE + STAGES;            // + V stage
  static constexpr int B_VE = B_VF + VSTAGES;
  static constexpr int B_SF = B_VE + VSTAGES;           // + tile
  static constexpr int B_PF = B_SF + 2;                 // P written, + 2 * tile + key half
  static constexpr int B_OD = B_PF + 4;                 // P.V done, + tile
  static constexpr int B_OE = B_OD + 2;                 // O read by the epilogue, + tile
  static constexpr int B_DRAIN = B_OE + 2;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // [0] TMEM base, [1] abort flag, [2] items
  // per-role stage counts compared at the end of the CTA (debug build):
  // [0] K/V stages loaded, [1] K/V stages consumed by the issuer, [2..3] P.V
  // products per tile, [4..5] score tiles the softmax warps processed per tile
  static constexpr int OFF_DBG = OFF_MISC + 16;
  // packed-sequence schedule: sequences sorted by row units (longest first),
  // per-unit-level sequence counts, and the first item of each level
  static constexpr int VL_MAX_SEQS = kVlMaxSeqs;
  static constexpr int VL_MAX_UNITS = kVlMaxUnits;
  static constexpr int OFF_VL = OFF_DBG + 32;                            // VarlenTables
  // packed kernel: a 32-row x 32-column O staging block (2 KB) per softmax
  // warp, over the schedule tables' build-time part (cnt, cur) and beyond
  static constexpr int OFF_OSTV = (OFF_VL + 4 * kVlCnt + 1023) / 1024 * 1024;
  static constexpr int BYTES_VL = OFF_VL + 4 * kVlInts > OFF_OSTV + 8 * 2048
                                      ? OFF_VL + 4 * kVlInts : OFF_OSTV + 8 * 2048;
  static constexpr int BYTES = VARLEN ? BYTES_VL : OFF_VL;
  static constexpr int SMEM_ALLOC = BYTES + 1024;       // slack for 1024-byte alignment
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 1);
};

// Division by a launch constant d without a divide: for 0 <= n < 2^31,
// n / d = umulhi(n, m) >> s with l = ceil(log2 d), m = ceil(2^(31 + l) / d) and
// s = l - 1 (Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994); m = 0 stands for d = 1.
struct FastDiv {
  uint32_t m, s;
};

__device__ __forceinline__ int fdiv(int n, FastDiv f) {
  return f.m ? int(__umulhi(uint32_t(n), f.m) >> f.s) : n;
}

struct FwdParams {
  void* o;                 // [B, Nq, Hq, D] bf16 or f32 (packed: [total_q, Hq, D])
  float* lse;              // [B, Hq, Nq] or null (packed: [Hq, total_q])
  int B, Hq, Hkv, Nq, Nk;  // packed: Nq, Nk are the longest sequence lengths
  // Packed variable-length sequences (kernel built with VARLEN): sequence b owns
  // query rows [cu_q[b], cu_q[b + 1]) of Q/O and keys [cu_k[b], cu_k[b + 1]) of K/V.
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  int nbh_seq;             // items per (sequence, row unit): n_bh / B
  int vl_hg;               // packed: heads (or head pairs) per group, divides nbh_seq
  int causal, window_left;
  float scale;             // softmax scale
  float scale_log2;        // scale * log2(e)
  int pair_heads;          // 1: tiles = two heads of a group at the same rows
  int n_qblk;              // ceil(Nq / 128)
  int n_units;             // row units per (b, head-or-pair)
  int n_bh;                // number of (b, head-or-pair) combinations
  int n_items;             // n_units * n_bh
  int hg;                  // equal lengths: (b, head-or-pair) per head group, divides n_bh
  int per_group;           // n_units * hg: items of one head group
  int bulk_o;              // equal-length bf16 O: 1 = staged bulk tensor stores, 0 = row stores
  // divisors of the item decode: hg, vl_hg, the (b, head-or-pair) combinations
  // per batch entry (Hkv * G/2 or Hq), and G/2 or G
  FastDiv fd_hg, fd_vlhg, fd_per_b, fd_inner;
};

constexpr int kFwdThreads = 384;
// Register split: the two softmax warpgroups hold a 128-score row each and
// take kFwdRegsSoftmax per thread; the issuer/producer warpgroup gives its
// registers up down to kFwdRegsOther. 192 / 120 uses the launch's 168 x 384
// registers exactly, and neither side spills (at 192 / 112 the issuer spills
// a few bytes once it walks the head-grouped work list). The launch must have
// at least kFwdRegsLaunchMin registers per thread for the split to fit; the
// host checks the built kernel's count.
#ifndef ATTN_REGS_SM
#define ATTN_REGS_SM 192
#endif
#ifndef ATTN_REGS_OT
#define ATTN_REGS_OT 120
#endif
constexpr int kFwdRegsSoftmax = ATTN_REGS_SM;
constexpr int kFwdRegsOther = ATTN_REGS_OT;
constexpr int kFwdRegsLaunch = 168;     // 65536 / 384 rounded down to a multiple of 8
constexpr int kFwdRegsLaunchMin = (2 * 128 * kFwdRegsSoftmax + 128 * kFwdRegsOther + kFwdThreads - 1) / kFwdThreads;
#ifndef ATTN_PROBE_REGS
static_assert(kFwdRegsLaunchMin <= kFwdRegsLaunch, "register split exceeds the launch budget");
#endif
// Every kPolyEvery-th pair of exponentials in an unmasked score tile is
// computed on the FMA pipe instead of the MUFU unit.
#ifndef ATTN_POLY_EVERY
#define ATTN_POLY_EVERY 8
#endif
constexpr int kPolyEvery = ATTN_POLY_EVERY;

struct TileInfo {
  int hq, row0, active;    // query head, first row, any row < nq
  int nq, nk;              // query rows and keys of this tile's sequence
  int blo, bhi;            // key blocks [blo, bhi); empty if bhi <= blo
};

__device__ __forceinline__ void tile_range(const FwdParams& p, TileInfo& t) {
  t.blo = 0;
  t.bhi = 0;
  if (!t.active) return;
  const int r_last = min(t.row0 + 127, t.nq - 1);
  const int qf = t.row0 + t.nk - t.nq;
  const int ql = r_last + t.nk - t.nq;
  const int hi = p.causal ? min(t.nk, ql + 1) : t.nk;
  const int lo = p.window_left >= 0 ? max(0, qf - p.window_left) : 0;
  if (hi <= lo) return;
  t.blo = lo / 128;
  t.bhi = (hi - 1) / 128 + 1;
}

__device__ __forceinline__ bool tile_has(const TileInfo& t, int j) {
  return j >= t.blo && j < t.bhi;
}

// Whether key block j needs element-wise masking for this tile's rows.
__device__ __forceinline__ bool block_needs_mask(const FwdParams& p, const TileInfo& t, int j) {
  const int kb0 = j * 128, kb1 = kb0 + 127;
  const int r_last = min(t.row0 + 127, t.nq - 1);
  const int qf = t.row0 + t.nk - t.nq;
  const int ql = r_last + t.nk - t.nq;
  return kb1 >= t.nk || (p.causal && kb1 > qf) || (p.window_left >= 0 && kb0 < ql - p.window_left);
}

// Both are called by the whole issuer warp (warp-uniform operands); one
// elected lane issues each MMA. The MMAs take descriptors built once per buffer: a descriptor's start
// address field is the byte address >> 4, so the descriptor of (address +
// off) is the buffer's descriptor + off >> 4 (off a multiple of 16 and the
// sum inside shared memory, which keeps the field below 2^14).
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc) {
  using L = FwdLayout<D>;
#pragma unroll
  for (int k = 0; k < D / 16; ++k) {
    const uint32_t off = ((k / 4) * L::HALF + (k % 4) * 32) >> 4;
    if (elect_one()) mma_ss(d_tmem, q_desc + off, k_desc + off, L::IDESC_QK, k > 0 ? 1u : 0u);
  }
}

// O += P V for keys [64 hf, 64 hf + 64) of the tile (four MMAs of 16 keys).
template <int D>
__device__ __forceinline__ void issue_pv_half(uint32_t d_tmem, uint32_t p_tmem, uint64_t v_desc,
                                              int hf, bool accumulate) {
  using L = FwdLayout<D>;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int k = 4 * hf + kk;
    if (elect_one())
      mma_ts(d_tmem, p_tmem + 8 * k, v_desc + ((k * 16 * 128) >> 4), L::IDESC_PV,
             (accumulate || k > 0) ? 1u : 0u);
  }
}

// One work item: a (batch, head-or-head-pair, row unit) and its two tiles.
struct WorkItem {
  int b, hkv;
  int q0, k0, bc;          // first Q row and first key of the sequence, batch coordinate
  TileInfo tile[2];
  int ubhi, U;             // key blocks visited: ubhi-1 down to ubhi-U
};

// Packed sequences: the work list holds only the items that exist. The heads
// (or head pairs) are taken in groups of vl_hg, one group after another, so the
// K/V of the items running at once fits in L2; within a group the rows run
// longest first. Sequences are sorted by their number of row units
// (descending), so at unit level u the sequences with more than u units are a
// prefix perm[0 .. cnt[u]) of the sorted order; level u's items start at
// lvl[u] within the group, and lvl[n_units] is the size of a group.

__device__ __forceinline__ int varlen_valid_rows(const FwdParams& p, int b) {
  const int q0 = __ldg(p.cu_q + b), q1 = __ldg(p.cu_q + b + 1);
  const int k0 = __ldg(p.cu_k + b), k1 = __ldg(p.cu_k + b + 1);
  const bool good = 0 <= q0 && q0 <= q1 && q1 <= p.total_q && q1 - q0 <= p.Nq &&
                    0 <= k0 && k0 <= k1 && k1 <= p.total_k && k1 - k0 <= p.Nk;
  return good ? q1 - q0 : -1;
}

__device__ __forceinline__ int varlen_units(const FwdParams& p, int nq) {
  const int per_unit = p.pair_heads ? 1 : 2;             // 128-row blocks per unit
  return nq <= 0 ? 0 : ((nq + 127) / 128 + per_unit - 1) / per_unit;
}

// Built by every thread of the CTA before the warp roles split (it ends with
// a CTA barrier); every CTA builds the same lists. Sequences with inconsistent
// offsets get no items and raise the status word.
__device__ void build_varlen_sched(const FwdParams& p, int* vl, int* n_items) {
  int* perm = vl;
  int* cnt = vl + kVlCnt;
  int* lvl = vl + kVlLvl;
  int* cur = vl + kVlCur;
  const int U = p.n_units;
  const int hg = p.vl_hg;                                // items per (sequence, unit, group)
  for (int u = threadIdx.x; u <= U; u += blockDim.x) cnt[u] = 0;
  __syncthreads();
  for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
    const int nq = varlen_valid_rows(p, b);
    if (nq < 0) atomicExch(&g_attn_status, kStatusBadInput);
    atomicAdd(&cnt[varlen_units(p, nq)], 1);             // histogram of unit counts
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // buckets laid out from U units down to 0: cnt[v] becomes the first slot of
    // bucket v, which is also the number of sequences with more than v units
    int slot = 0;
    for (int v = U; v >= 0; --v) {
      const int h = cnt[v];
      cnt[v] = slot;
      cur[v] = slot;
      slot += h;
    }
    // levels within one head group; the groups repeat the pattern
    int item = 0;
    for (int u = U - 1; u >= 0; --u) {
      lvl[u] = item;
      item += cnt[u] * hg;
    }
    lvl[U] = item;                                       // items of one head group
    *n_items = item * (p.nbh_seq / hg);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < p.B; b += blockDim.x)
    perm[atomicAdd(&cur[varlen_units(p, varlen_valid_rows(p, b))], 1)] = b;
  __syncthreads();
}

// vl: the packed-sequence tables (null for the closed-form work list).
template <bool VARLEN>
__device__ __forceinline__ void decode_item(const FwdParams& p, int g, int ig, WorkItem& w,
                                            const int* vl) {
  // item ig of head group g
  int unit, bh;
  if constexpr (VARLEN) {
    const int* lvl = vl + kVlLvl;
    // level: the lowest u whose first item is <= the item's index within the
    // group (lvl grows as u falls)
    int lo = 0, hi = p.n_units - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (lvl[mid] <= ig) hi = mid; else lo = mid + 1;
    }
    unit = lo;
    const int r = ig - lvl[unit];
    const int s = fdiv(r, p.fd_vlhg);
    bh = vl[s] * p.nbh_seq + g * p.vl_hg + (r - s * p.vl_hg);
  } else {
    // head groups one after another (so the K/V the running items touch stays
    // in L2), the longest rows first within a group
    const int lvl = fdiv(ig, p.fd_hg);
    unit = p.n_units - 1 - lvl;
    bh = g * p.hg + (ig - lvl * p.hg);
  }
  if (p.pair_heads) {
    const int G = p.Hq / p.Hkv;
    const int pairs = G / 2;
    w.b = fdiv(bh, p.fd_per_b);
    const int rem = bh - w.b * (p.Hkv * pairs);
    w.hkv = fdiv(rem, p.fd_inner);
    const int pr = rem - w.hkv * pairs;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      w.tile[t].hq = w.hkv * G + 2 * pr + t;
      w.tile[t].row0 = unit * 128;
    }
  } else {
    w.b = fdiv(bh, p.fd_per_b);
    const int hq = bh - w.b * p.Hq;
    w.hkv = fdiv(hq, p.fd_inner);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      w.tile[t].hq = hq;
      w.tile[t].row0 = (2 * unit + t) * 128;
    }
  }
  int nq = p.Nq, nk = p.Nk;
  w.q0 = 0;
  w.k0 = 0;
  w.bc = w.b;
  if constexpr (VARLEN) {
    // sequence bounds from the offsets; an inconsistent sequence (outside the
    // packed tensors, or longer than the longest length the host gave) is
    // skipped and flagged, so nothing is written outside O and LSE
    const int q0 = __ldg(p.cu_q + w.b), q1 = __ldg(p.cu_q + w.b + 1);
    const int k0 = __ldg(p.cu_k + w.b), k1 = __ldg(p.cu_k + w.b + 1);
    const bool good = 0 <= q0 && q0 <= q1 && q1 <= p.total_q && q1 - q0 <= p.Nq &&
                      0 <= k0 && k0 <= k1 && k1 <= p.total_k && k1 - k0 <= p.Nk;
    if (!good) atomicExch(&g_attn_status, kStatusBadInput);
    nq = good ? q1 - q0 : 0;
    nk = good ? k1 - k0 : 0;
    w.q0 = good ? q0 : 0;
    w.k0 = good ? k0 : 0;
    w.bc = 0;
  }
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    w.tile[t].nq = nq;
    w.tile[t].nk = nk;
    w.tile[t].active = w.tile[t].row0 < nq;
    tile_range(p, w.tile[t]);
  }
  const bool ne0 = w.tile[0].bhi > w.tile[0].blo, ne1 = w.tile[1].bhi > w.tile[1].blo;
  int ublo = 0, ubhi = 0;
  if (ne0 || ne1) {
    ublo = ne0 ? (ne1 ? min(w.tile[0].blo, w.tile[1].blo) : w.tile[0].blo) : w.tile[1].blo;
    ubhi = ne0 ? (ne1 ? max(w.tile[0].bhi, w.tile[1].bhi) : w.tile[0].bhi) : w.tile[1].bhi;
  }
  w.ubhi = ubhi;
  w.U = ubhi - ublo;
}

// This CTA's work items, in order. The list is a sequence of head groups of
// per_group items, the longest rows first within a group. A group's items go
// to the CTAs in a boustrophedon (close to a longest-processing-time
// schedule) that starts at the CTA where the previous group's items ended, so
// the group boundaries do not pile every group's long items onto the same
// CTAs. With one group this is the plain boustrophedon over the whole list.
struct ItemCursor {
  int g = 0, k = 0;                        // group, this CTA's position within it
  int start = 0;                           // first CTA of group g: g * per_group mod grid
};

// The index within group cur.g of this CTA's next item, or -1 when none is
// left. pg_mod = per_group mod the grid size.
__device__ __forceinline__ int next_item(ItemCursor& cur, int per_group, int n_groups, int pg_mod) {
  const int G = int(gridDim.x);
  while (cur.g < n_groups) {
    const int c0 = int(blockIdx.x) - cur.start;
    const int c = c0 < 0 ? c0 + G : c0;
    const long long i = static_cast<long long>(cur.k) * G + ((cur.k & 1) ? G - 1 - c : c);
    if (i < per_group) {
      ++cur.k;
      return int(i);
    }
    ++cur.g;
    cur.k = 0;
    cur.start += pg_mod;
    if (cur.start >= G) cur.start -= G;
  }
  return -1;
}

template <int D, bool F32OUT, bool VARLEN>
__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                const FwdParams p) {
  using L = FwdLayout<D, VARLEN>;
  // bf16 O of the equal-length kernel leaves through shared memory and bulk
  // tensor stores (tmO) when p.bulk_o, which the host sets for every bf16
  // launch; otherwise each thread stores its row from registers. The choice
  // stays a launch parameter: built that way, the kernel measured 1-3 points
  // of the bf16 peak faster than with the bulk stores fixed at compile time.
  constexpr bool kTmaO = !VARLEN && !F32OUT;
  // the packed kernel stores O the same way from the warps whose 32 rows all
  // lie inside their sequence, through 2 KB blocks of 32 columns
  constexpr bool kTmaOV = VARLEN && !F32OUT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::OFF_BAR + 8u * uint32_t(i); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- setup ---------------------------------------------------------------
  if (threadIdx.x == 0) {
    mbar_init(bar(L::B_Q), 1);
    mbar_init(bar(L::B_QE), 1);
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(bar(L::B_KF + s), 1);
      mbar_init(bar(L::B_KE + s), 1);
    }
    for (int s = 0; s < L::VSTAGES; ++s) {
      mbar_init(bar(L::B_VF + s), 1);
      mbar_init(bar(L::B_VE + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::B_SF + t), 1);
      mbar_init(bar(L::B_PF + 2 * t + 0), 128);
      mbar_init(bar(L::B_PF + 2 * t + 1), 128);
      mbar_init(bar(L::B_OD + t), 1);
      mbar_init(bar(L::B_OE + t), 128);
    }
    mbar_init(bar(L::B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_holder), L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // the work list: closed form, or the compact list of packed sequences
  const int* vs = nullptr;
  int per_group = p.per_group, n_groups = p.n_bh / p.hg;
  if constexpr (VARLEN) {
    int* vl = reinterpret_cast<int*>(smem + L::OFF_VL);
    int* vl_items = reinterpret_cast<int*>(smem + L::OFF_MISC + 8);
    build_varlen_sched(p, vl, vl_items);
    vs = vl;
    per_group = vl[kVlLvl + p.n_units];                 // items of one head group
    n_groups = p.nbh_seq / p.vl_hg;
  }
  const int pg_mod = per_group % int(gridDim.x);

  if (warp < 8) {
    // ======================= softmax warpgroups ==============================
    reg_alloc<kFwdRegsSoftmax>();
    const int t = warp >> 2;
    const int row = int(threadIdx.x) - 128 * t;
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + (t ? L::COL_S1 : L::COL_S0);
    const uint32_t tO = tmem + lane_off + (t ? L::COL_O1 : L::COL_O0);
    const float c2 = p.scale_log2;
    int count = 0;                          // S tiles processed so far (all items)
    bool ok = true;
    ItemCursor cur;
    while (ok) {
      const int ig = next_item(cur, per_group, n_groups, pg_mod);
      if (ig < 0) break;
      WorkItem w;
      decode_item<VARLEN>(p, cur.g, ig, w, vs);
      const TileInfo T = t ? w.tile[1] : w.tile[0];   // by value: no local-memory copy of w
      if (!T.active) continue;
      const int r = T.row0 + row;
      const int qpos = r + T.nk - T.nq;
      float m = -CUDART_INF_F;              // running max (raw score units)
      float l = 0.f;                        // running sum of exp2((s - m) * c2)
      int n_in_item = 0;
      for (int j = T.bhi - 1; j >= T.blo; --j) {
        // S_t(j) is issued after this tile's previous P.V and its commit covers
        // every earlier MMA of the issuer, so once S is ready the previous P.V
        // has completed: P may be overwritten and O rescaled.
        const bool wt = mbar_wait<1>(bar(L::B_SF + t), uint32_t(count & 1), abort_flag);
        if (!__all_sync(0xffffffffu, wt)) { ok = false; break; }
        tc_fence_after();

        uint32_t sr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, sr + 32 * c);
        tmem_wait_ld();
        float s[128];
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);

        const bool masked = block_needs_mask(p, T, j);
        if (masked) {
          // allowed keys of this row, relative to the block: [lo_rel, hi_rel]
          const int kb0 = j * 128;
          int hi = T.nk - 1;
          if (p.causal) hi = min(hi, qpos);
          int lo = 0;
          if (p.window_left >= 0) lo = qpos - p.window_left;
          const int lo_rel = lo - kb0, hi_rel = hi - kb0;
          // 32-key chunks that every row of the warp may see in full skip the
          // compares (the choice is warp-uniform); on a causal diagonal block
          // warp w has w such chunks.
          const int lo_max = __reduce_max_sync(0xffffffffu, lo_rel);
          const int hi_min = __reduce_min_sync(0xffffffffu, hi_rel);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (32 * q < lo_max || 32 * q + 31 > hi_min) {
              if (p.window_left >= 0) {
#pragma unroll
                for (int c = 32 * q; c < 32 * q + 32; ++c)
                  if (c < lo_rel || c > hi_rel) s[c] = -CUDART_INF_F;
              } else {                        // no window: lo_rel <= 0
#pragma unroll
                for (int c = 32 * q; c < 32 * q + 32; ++c)
                  if (c > hi_rel) s[c] = -CUDART_INF_F;
              }
            }
          }
        }
        // row max: 8 independent chains of three-input maxima
        float mx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = max3f(s[i], s[8 + i], s[16 + i]);
#pragma unroll
        for (int c = 24; c < 120; c += 16) {
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = max3f(mx[i], s[c + i], s[c + 8 + i]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], s[120 + i]);
        const float mb = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]),
                               fmaxf(mx[6], mx[7]));
        // Lazy rescale: keep the old maximum while the new one exceeds it by at
        // most 8 in log2 units (P values stay <= 256); the final O / l is exact
        // whichever maximum was used.
        const float m_new = fmaxf(m, mb);
        const bool rescale = (m_new - m) * c2 > 8.0f;     // false when both are -inf
        float alpha = 1.f;
        if (rescale) {
          alpha = ex2_approx((m - m_new) * c2);            // 0 when m was -inf
          m = m_new;
        }
        const float mo = (m == -CUDART_INF_F) ? 0.f : m * c2;
        // P = 2^(s * c2 - mo) on pairs; in unmasked tiles every kPolyEvery-th
        // pair goes to the FMA-pipe polynomial to offload the MUFU unit. P is
        // written and announced in two halves of 64 keys so the tensor core
        // starts P.V on the first half while the second is computed.
        const uint64_t C2 = f2_pack(c2, c2), NMO = f2_pack(-mo, -mo);
        uint64_t lacc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[32];
          if (masked) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int c = 32 * hf + i;
              const float2 x = f2_unpack(f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), C2, NMO));
              const float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
              lacc[i & 3] = f2_add(lacc[i & 3], f2_pack(p0, p1));
              pk[i] = pack_bf16x2(p0, p1);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int c = 32 * hf + i;
              float p0, p1;
              if ((i % kPolyEvery) == kPolyEvery - 1) {
                const uint64_t x = f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), C2, NMO);
                const float2 ee = f2_unpack(exp2_poly_f2(x));
                p0 = ee.x;
                p1 = ee.y;
              } else {
                const float2 xx = f2_unpack(f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), C2, NMO));
                p0 = ex2_approx(xx.x);
                p1 = ex2_approx(xx.y);
              }
              lacc[i & 3] = f2_add(lacc[i & 3], f2_pack(p0, p1));
              pk[i] = pack_bf16x2(p0, p1);
            }
          }
          tmem_st32(tS + 32 * hf, pk);
          if (hf == 0 && n_in_item > 0 && __any_sync(0xffffffffu, rescale)) {
            // O must be rescaled before the first half's P.V accumulates
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tO + 32 * c, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tO + 32 * c, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(L::B_PF + 2 * t + hf));
        }
        const float2 l01 = f2_unpack(f2_add(f2_add(lacc[0], lacc[1]), f2_add(lacc[2], lacc[3])));
        const float lsum = l01.x + l01.y;
        l = fmaf(l, alpha, lsum);
        ++count;
        ++n_in_item;
      }
      if (!ok) break;

      // ---- epilogue: O / l and LSE -----------------------------------------
      // LSE first: it needs only m and l, so its store overlaps the wait for
      // the last P.V
      const long long o_rows = VARLEN ? p.total_q : static_cast<long long>(p.B) * p.Nq;
      const bool row_ok = r < T.nq &&
                          in_bounds(VARLEN ? w.q0 + r : static_cast<long long>(w.b) * p.Nq + r, o_rows) &&
                          in_bounds(T.hq, p.Hq);
      if (row_ok && p.lse != nullptr) {
        const size_t li = VARLEN ? size_t(T.hq) * p.total_q + w.q0 + r : (size_t(w.b) * p.Hq + T.hq) * p.Nq + r;
        if (in_bounds(static_cast<long long>(li), static_cast<long long>(p.Hq) * o_rows))
          p.lse[li] = (l > 0.f) ? fmaf(m, p.scale, __log2f(l) * 0.6931471805599453f) : -CUDART_INF_F;
      }
      bool have = n_in_item > 0;
      if (have) {
        const bool wt = mbar_wait<1>(bar(L::B_OD + t), uint32_t((count - 1) & 1), abort_flag);
        if (!__all_sync(0xffffffffu, wt)) { ok = false; break; }
        tc_fence_after();
      }
      uint32_t o[D];
      if (have) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + 32 * c, o + 32 * c);
        tmem_wait_ld();
        // O of this tile has been read: the next item's first P.V may overwrite it
        tc_fence_before();
        mbar_arrive(bar(L::B_OE + t));
      } else {
#pragma unroll
        for (int e = 0; e < D; ++e) o[e] = 0u;
      }
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      const bool bulk_o = (kTmaO || kTmaOV) && p.bulk_o;
      const int wr0 = T.row0 + 32 * (warp & 3);
      const bool warp_bulk = bulk_o && (VARLEN ? wr0 + 32 <= T.nq : wr0 < T.nq);
      if constexpr (kTmaOV) {
        if (warp_bulk) {
          // 32 columns at a time: 64-byte rows with the 64-byte swizzle of the
          // tensor map; the block is rewritten after its previous store read it
          const uint32_t stg = sb + L::OFF_OSTV + uint32_t(warp) * 2048u;
          const uint32_t rb = stg + uint32_t(lane) * 64u;
#pragma unroll
          for (int qc = 0; qc < D / 32; ++qc) {
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint32_t* e = o + 32 * qc + 8 * c;
              st_shared_v4(rb + uint32_t((c ^ ((lane >> 1) & 3)) << 4),
                           pack_bf16x2(__uint_as_float(e[0]) * inv, __uint_as_float(e[1]) * inv),
                           pack_bf16x2(__uint_as_float(e[2]) * inv, __uint_as_float(e[3]) * inv),
                           pack_bf16x2(__uint_as_float(e[4]) * inv, __uint_as_float(e[5]) * inv),
                           pack_bf16x2(__uint_as_float(e[6]) * inv, __uint_as_float(e[7]) * inv));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && in_bounds(T.hq, p.Hq) &&
                in_bounds(static_cast<long long>(w.q0) + wr0 + 31, static_cast<long long>(p.total_q))) {
              tma_store_4d(&tmO, stg, 32 * qc, T.hq, w.q0 + wr0, 0);
              bulk_commit_group();
            }
          }
        }
      }
      if (kTmaO && warp_bulk) {
        // Each warp writes its 32 rows to its own staging block, 64 columns at
        // a time, in the 128-byte swizzled layout of the tensor map; lane 0
        // then stores the block (rows past Nq fall outside the map and are not
        // written). A block is rewritten only after its previous store has
        // read it. Only warp-level synchronisation: no warp ever waits on
        // another one here.
        {
          const uint32_t stg = sb + L::OFF_OST + uint32_t(t) * L::HALF + uint32_t(warp & 3) * 4096u;
          const uint32_t rbase = stg + uint32_t(lane) * 128u;
#pragma unroll
          for (int h = 0; h < D / 64; ++h) {
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint32_t* e = o + 64 * h + 8 * c;
              st_shared_v4(rbase + uint32_t((c ^ (lane & 7)) << 4),
                           pack_bf16x2(__uint_as_float(e[0]) * inv, __uint_as_float(e[1]) * inv),
                           pack_bf16x2(__uint_as_float(e[2]) * inv, __uint_as_float(e[3]) * inv),
                           pack_bf16x2(__uint_as_float(e[4]) * inv, __uint_as_float(e[5]) * inv),
                           pack_bf16x2(__uint_as_float(e[6]) * inv, __uint_as_float(e[7]) * inv));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && in_bounds(w.b, p.B) && in_bounds(T.hq, p.Hq)) {
              tma_store_4d(&tmO, stg, 64 * h, T.hq, wr0, w.b);
              bulk_commit_group();
            }
          }
        }
      }
      if (row_ok) {
        const size_t orow = VARLEN ? size_t(w.q0) + r : size_t(w.b) * p.Nq + r;
        const size_t obase = (orow * p.Hq + T.hq) * D;
        if constexpr (F32OUT) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + obase);
#pragma unroll
          for (int e = 0; e < D / 4; ++e)
            dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                                 __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
        } else if (!warp_bulk) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + obase);
#pragma unroll
          for (int e = 0; e < D / 8; ++e) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * e + 0]) * inv, __uint_as_float(o[8 * e + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv);
            dst[e] = v;
          }
        }
      }
    }
    // the CTA's shared memory must outlive the last O stores
    if ((kTmaO || kTmaOV) && lane == 0) bulk_wait_all();
    if (row == 0) reinterpret_cast<volatile int*>(smem + L::OFF_DBG)[4 + t] = count;
  } else {
  // warps 8-11 release registers to the softmax warpgroups (the release is
  // larger than the softmax groups' increase)
  reg_dealloc<kFwdRegsOther>();
  if (warp == 8) {
    // ======================= tensor-core issuer ==============================
    // The whole warp runs the loop, so every operand is warp-uniform; one
    // elected lane (always lane 0) issues each MMA and commit.
    {
      // a wait the whole warp agrees on (lanes give up together)
      auto wwait = [&](int b, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar(b), parity, abort_flag));
      };
      auto commit = [&](int b) { if (elect_one()) tc_commit(bar(b)); };
      const uint64_t dq0 = smem_desc_sw128(sb + L::OFF_Q, 16, 1024);
      const uint64_t dq1 = smem_desc_sw128(sb + L::OFF_Q + L::TILE, 16, 1024);
      const uint64_t dk = smem_desc_sw128(sb + L::OFF_K, 16, 1024);          // + slot * TILE
      const uint64_t dv = smem_desc_sw128(sb + L::OFF_V, L::HALF, 1024);     // + slot * TILE
      const uint32_t dS0 = tmem + L::COL_S0, dS1 = tmem + L::COL_S1;
      const uint32_t dO0 = tmem + L::COL_O0, dO1 = tmem + L::COL_O1;
      int pv[2] = {0, 0};                   // P.V products issued per tile (all items)
      int done[2] = {0, 0};                 // items in which each tile had work
      bool first[2] = {true, true};         // no P.V of the tile yet in this item
      // O_t += P_t V: each 64-key half as soon as the softmax has written it
      auto pv_tile = [&](int t, int vslot) -> bool {
        const uint64_t vd = dv + uint32_t(vslot * (L::TILE >> 4));
        const uint32_t dO = t ? dO1 : dO0, dS = t ? dS1 : dS0;
        if (!wwait(L::B_PF + 2 * t + 0, uint32_t(pv[t] & 1))) return false;
        if (first[t] && done[t] > 0 &&
            !wwait(L::B_OE + t, uint32_t((done[t] - 1) & 1))) return false;
        tc_fence_after();
        issue_pv_half<D>(dO, dS, vd, 0, !first[t]);
        if (!wwait(L::B_PF + 2 * t + 1, uint32_t(pv[t] & 1))) return false;
        tc_fence_after();
        issue_pv_half<D>(dO, dS, vd, 1, true);
        commit(L::B_OD + t);
        ++pv[t];
        first[t] = false;
        return true;
      };
      int kv = 0, qi = 0;                   // K/V ring position, items with a Q load
      bool alive = true;
      ItemCursor cur;
      while (alive) {
        const int ig = next_item(cur, per_group, n_groups, pg_mod);
        if (ig < 0) break;
        WorkItem w;
        decode_item<VARLEN>(p, cur.g, ig, w, vs);
        if (w.U == 0) continue;
        if (!(alive = wwait(L::B_Q, uint32_t(qi & 1)))) break;
        tc_fence_after();
        first[0] = first[1] = true;
        int prev_j = -1, prev_vslot = 0;
        for (int it = 0; it < w.U; ++it, ++kv) {
          const int j = w.ubhi - 1 - it;
          const int slot = kv % L::STAGES;
          const uint32_t ph = uint32_t(kv / L::STAGES) & 1u;
          const int vslot = kv % L::VSTAGES;
          const uint32_t vph = uint32_t(kv / L::VSTAGES) & 1u;
          if (!(alive = wwait(L::B_KF + slot, ph))) break;
          tc_fence_after();
          const uint64_t kd = dk + uint32_t(slot * (L::TILE >> 4));
          if (tile_has(w.tile[0], j)) {
            issue_qk<D>(dS0, dq0, kd);
            commit(L::B_SF + 0);
          }
          if (it > 0) {
            if (tile_has(w.tile[1], prev_j) && !(alive = pv_tile(1, prev_vslot))) break;
            commit(L::B_VE + prev_vslot);
          }
          if (tile_has(w.tile[1], j)) {
            issue_qk<D>(dS1, dq1, kd);
            commit(L::B_SF + 1);
          }
          commit(L::B_KE + slot);
          if (it == w.U - 1) commit(L::B_QE);     // every Q.K^T of this item issued
          if (!(alive = wwait(L::B_VF + vslot, vph))) break;
          tc_fence_after();
          if (tile_has(w.tile[0], j) && !(alive = pv_tile(0, vslot))) break;
          prev_j = j;
          prev_vslot = vslot;
        }
        if (!alive) break;
        if (tile_has(w.tile[1], prev_j) && !(alive = pv_tile(1, prev_vslot))) break;
        commit(L::B_VE + prev_vslot);
        if (!first[0]) ++done[0];
        if (!first[1]) ++done[1];
        ++qi;
      }
      // drain: every issued tensor-core operation completes before teardown
      commit(L::B_DRAIN);
      mbar_wait(bar(L::B_DRAIN), 0, nullptr);
      __syncwarp();
      if (lane == 0) {
        volatile int* dbg = reinterpret_cast<volatile int*>(smem + L::OFF_DBG);
        dbg[1] = kv;
        dbg[2] = pv[0];
        dbg[3] = pv[1];
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ======================= TMA producer ====================================
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int kv = 0, qi = 0;                   // same counters as the issuer
      int issued_k = 0, issued_v = 0;
      bool alive = true;
      ItemCursor cur;
      while (alive) {
        const int ig = next_item(cur, per_group, n_groups, pg_mod);
        if (ig < 0) break;
        WorkItem w;
        decode_item<VARLEN>(p, cur.g, ig, w, vs);
        if (w.U == 0) continue;
        // Q buffers are free once every Q.K^T of the previous item completed
        if (qi > 0 && !(alive = mbar_wait(bar(L::B_QE), uint32_t((qi - 1) & 1), abort_flag))) break;
        mbar_arrive_expect_tx(bar(L::B_Q), 2 * L::TILE);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          // an active tile's first row lies inside Q (an inactive one reads
          // zeros past the end, which is what the copy engine gives there)
          if (w.tile[t].active) {
            (void)in_bounds(w.q0 + w.tile[t].row0, VARLEN ? p.total_q : p.Nq);
            (void)in_bounds(w.tile[t].hq, p.Hq);
          }
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sb + L::OFF_Q + t * L::TILE + c * L::HALF, &tmQ, bar(L::B_Q), c * 64,
                        w.tile[t].hq, w.q0 + w.tile[t].row0, w.bc);
        }
        (void)in_bounds(w.bc, VARLEN ? 1 : p.B);
        (void)in_bounds(w.hkv, p.Hkv);
        ++qi;
        for (int it = 0; it < w.U; ++it, ++kv) {
          const int j = w.ubhi - 1 - it;
          const int slot = kv % L::STAGES;
          const uint32_t ph = uint32_t(kv / L::STAGES) & 1u;
          if (!(alive = mbar_wait(bar(L::B_KE + slot), ph ^ 1u, abort_flag))) break;
          (void)in_bounds(w.k0 + j * 128, VARLEN ? p.total_k : p.Nk);   // the tile's first key
          mbar_arrive_expect_tx(bar(L::B_KF + slot), L::TILE);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sb + L::OFF_K + slot * L::TILE + c * L::HALF, &tmK, bar(L::B_KF + slot),
                        c * 64, w.hkv, w.k0 + j * 128, w.bc);
          issued_k = kv + 1;
          const int vslot = kv % L::VSTAGES;
          const uint32_t vph = uint32_t(kv / L::VSTAGES) & 1u;
          if (!(alive = mbar_wait(bar(L::B_VE + vslot), vph ^ 1u, abort_flag))) break;
          mbar_arrive_expect_tx(bar(L::B_VF + vslot), L::TILE);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sb + L::OFF_V + vslot * L::TILE + c * L::HALF, &tmV, bar(L::B_VF + vslot),
                        c * 64, w.hkv, w.k0 + j * 128, w.bc);
          issued_v = kv + 1;
        }
      }
      // Make sure no copy is still landing in shared memory at exit: wait for
      // the most recent phase of every stage (already complete normally).
      if (qi > 0) mbar_wait(bar(L::B_Q), uint32_t((qi - 1) & 1), nullptr);
      for (int it = max(0, issued_k - L::STAGES); it < issued_k; ++it)
        mbar_wait(bar(L::B_KF + it % L::STAGES), uint32_t(it / L::STAGES) & 1u, nullptr);
      for (int it = max(0, issued_v - L::VSTAGES); it < issued_v; ++it)
        mbar_wait(bar(L::B_VF + it % L::VSTAGES), uint32_t(it / L::VSTAGES) & 1u, nullptr);
      reinterpret_cast<volatile int*>(smem + L::OFF_DBG)[0] = issued_v;
    }
    __syncwarp();
  }
  }

  // ---- teardown --------------------------------------------------------------
  // (register budgets stay split: no warpgroup increases its budget again, so
  // the only increase, the softmax groups' at the start, is always granted)
  tc_fence_before();
  __syncthreads();
  if (kDebugBounds && threadIdx.x == 0 && *abort_flag == 0) {
    // every role walked the same stages: loads = issues, P.V products = score
    // tiles the softmax warps processed, per tile
    const volatile int* dbg = reinterpret_cast<const volatile int*>(smem + L::OFF_DBG);
    (void)(same_count(dbg[0], dbg[1]) && same_count(dbg[2], dbg[4]) && same_count(dbg[3], dbg[5]));
  }
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace attn
