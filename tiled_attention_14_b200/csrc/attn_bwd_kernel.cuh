// attn_bwd_kernel.cuh — fused attention backward for sm_100a (B200).
//
// What it computes: the gradients dQ, dK, dV of the attention forward (same score_mod and
// masks, grouped-query heads included) from Q, K, V, O, dO and the forward's per-row
// log-sum-exp, so that neither P nor dP ever reaches HBM.  The pages compare FA4's
// backward passes with cuDNN's and warn that block-sparse backward runs are not
// deterministic (page "PyTorch's FlexAttention mit FlashAttention-4 ist ein Game-Changer",
// sections "Leistung und Validierung" and "Aktuelle Einschränkungen"); the page
// "FlashAttention 4: ..." lists the backward among FA4's missing parts (section "Κύρια
// Συμπεράσματα").  With t = score_mod(scale * q.k) and P = exp(t - LSE):
//     dV = P^T dO,  dP = dO V^T,  dS = P * (dP - Dv) * dt/ds,  Dv_i = sum_d dO_id O_id,
//     dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Deterministic by construction: no floating-point atomics.  Three launches:
//   attn_bwd_prep_kernel   Dv and LSE * log2(e) per query row, padded to 128-row tiles
//                          (plus a "document ids sorted" flag per batch row)
//   attn_bwd_dkdv_kernel   one work item = one 128-key tile of one key/value head; it walks
//                          every (query head of the group, 128-row query tile) that sees the
//                          tile, accumulating dV and dK in tensor memory in a fixed order
//   attn_bwd_dq_kernel     one work item = one 128-row query tile of one head; it walks the
//                          visible key tiles, accumulating dQ in tensor memory
// dQ is computed apart from dK/dV (recomputing S and dP) instead of being summed across
// CTAs, which is what keeps the result bit-reproducible.
//
// Each kernel: 10 warps — warps 0-7 compute (two per TMEM lane quarter, one half of the 128
// columns each), warp 8 issues the TMA loads, one thread of warp 9 issues the MMAs.
// Tensor memory, dK/dV kernel: S^T | dP^T | dV | dK (P^T and dS^T in bf16 over the first
// columns of S^T and dP^T); dQ kernel: S | dP_0 | dP_1 | dQ (dP double-buffered, dS in bf16
// over the dP it came from).  The hand-offs are split so that the tensor core works while the
// compute warps do: in the dK/dV kernel dV and the next S^T run during the dS pass, dK and
// the next dP^T during the next P pass; in the dQ kernel the next S is computed as soon as
// this step's S has been read and the dP two steps ahead right after dQ, so that a step never
// waits for the tensor core.
// Every wait is bounded as in the forward kernel.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "attn_fwd_kernel.cuh"

namespace attn {

// 10 warps: 0-7 compute (warps w and w+4 share the TMEM lane quarter w % 4 = 32 rows of the
// tile and take one half of its 128 columns each), 8 issues the TMA loads, one thread of 9
// issues the MMAs.
constexpr int kBwdThreads = 320;
constexpr int kBwdCompute = 256;
constexpr int kBwdLoadWarp = 8;
constexpr int kBwdMmaWarp = 9;

struct BwdParams {
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const float* lse2;       // [B*H, Sq_pad]: LSE * log2(e); +inf for rows without keys and padding
  const float* dvec;       // [B*H, Sq_pad]: sum_d dO * O; 0 for padding
  int B, H, Hkv, group, Sq, Sk, Sq_pad;
  int nqt, nkt;            // 128-row query tiles, 128-key tiles
  int mask_kind, window;
  float scale;             // scale of the scores (dQ and dK are multiplied by it at the end)
  float scale_log2;        // scale * log2(e)
  float sc_in, sc_out;     // soft-capping: th = tanh(s * sc_in), t = th * sc_out (log2 units)
  const float* alibi;      // [H] or nullptr
  const int* doc;          // [B, Sk] or nullptr
  const int* doc_sorted;   // [B] flags (from the prep kernel) or nullptr
  int num_items;
  int lpt;                 // causal: longest items first
  unsigned long long timeout_ns;
};

template <int D>
struct BwdCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;         // one 128-row bf16 tile
  static constexpr int PANEL_BYTES = 128 * 128;
  static constexpr int NPANEL = D / 64;
  static constexpr int NST = 2;                          // streamed-tile ring depth
  // dK/dV kernel: K | V | NST x (Q | dO) | NST x (lse2 | dvec) ; dQ kernel: Q | dO | NST x (K | V)
  static constexpr int OFF_A = 0;                        // K (dkdv) or Q (dq)
  static constexpr int OFF_B = TILE_BYTES;               // V (dkdv) or dO (dq)
  static constexpr int OFF_RING = 2 * TILE_BYTES;        // stage s: [OFF_RING + s*2*TILE, +TILE)
  static constexpr int OFF_ROWS = OFF_RING + NST * 2 * TILE_BYTES;   // NST x 1 KB (lse2, dvec)
  static constexpr int OFF_BAR = OFF_ROWS + NST * 1024;
  static constexpr int NBAR = 20;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // At least 120 KB so that two CTAs never share an SM: each allocates all 512 TMEM
  // columns, and a second CTA on the SM would wait for the first one's to be freed.
  static constexpr int SMEM_USED = OFF_MISC + 16 + 1024;
  static constexpr int SMEM_BYTES = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 0, T_DP = 128, T_ACC0 = 256, T_ACC1 = 256 + D;
  // dQ kernel: S, two dP buffers (dS is written over the dP it came from), dQ
  static constexpr uint32_t T_DP0 = 128, T_DP1 = 256, T_DQ = 384;
  // dQ kernel shared memory: Q | dO | K ring | V ring.  K is read by S one step ahead and by
  // dQ at the end of its step; V only by dP, two steps ahead: so K gets three slots and V two,
  // which lets every slot be reloaded a full step before it is needed.
  static constexpr int DQ_NK = 3, DQ_NV = 2;
  static constexpr int DQ_OFF_K = 2 * TILE_BYTES;
  static constexpr int DQ_OFF_V = DQ_OFF_K + DQ_NK * TILE_BYTES;
  static constexpr int DQ_OFF_BAR = DQ_OFF_V + DQ_NV * TILE_BYTES;
  static constexpr int DQ_OFF_MISC = DQ_OFF_BAR + NBAR * 8;
  static constexpr int DQ_SMEM_USED = DQ_OFF_MISC + 16 + 1024;
  static constexpr int DQ_SMEM_BYTES = DQ_SMEM_USED > 120 * 1024 ? DQ_SMEM_USED : 120 * 1024;
  static_assert(DQ_SMEM_BYTES <= 227 * 1024, "dQ kernel shared memory");
  static constexpr uint32_t IDESC_SS = make_idesc(1u, 128, 128, false);   // 128x128, both K-major
  static constexpr uint32_t IDESC_TS = make_idesc(1u, 128, D, true);      // A from TMEM, B MN-major
};

// ---------------------------------------------------------------------------------------
// preparation: Dv = rowsum(dO * O), LSE in log2 units, padded to whole 128-row tiles
// ---------------------------------------------------------------------------------------
constexpr int kPrepThreads = 256;   // 8 warps, one query row per warp at a time

template <int D>
__global__ void __launch_bounds__(kPrepThreads)
attn_bwd_prep_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                     const float* __restrict__ lse, float* __restrict__ lse2, float* __restrict__ dvec,
                     int Sq, int Sq_pad, long long rows_total) {
  const int lane = threadIdx.x & 31;
  const long long warp_g = (static_cast<long long>(blockIdx.x) * kPrepThreads + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * kPrepThreads) >> 5;
  for (long long r = warp_g; r < rows_total; r += nwarps) {   // r over (bh, row < Sq_pad)
    const long long bh = r / Sq_pad;
    const int row = static_cast<int>(r - bh * Sq_pad);
    float dsum = 0.f, l2 = __builtin_huge_valf();
    if (row < Sq) {
      const size_t base = (static_cast<size_t>(bh) * Sq + row) * D;
      constexpr int PER = D / 32;   // elements per lane (2 or 4)
      if constexpr (PER == 4) {
        const uint2 a = *reinterpret_cast<const uint2*>(o + base + lane * 4);
        const uint2 b = *reinterpret_cast<const uint2*>(dout + base + lane * 4);
        const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a.x));
        const float2 a1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a.y));
        const float2 b0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b.x));
        const float2 b1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b.y));
        dsum = a0.x * b0.x + a0.y * b0.y + a1.x * b1.x + a1.y * b1.y;
      } else {
        const uint32_t a = *reinterpret_cast<const uint32_t*>(o + base + lane * 2);
        const uint32_t b = *reinterpret_cast<const uint32_t*>(dout + base + lane * 2);
        const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a));
        const float2 b0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b));
        dsum = a0.x * b0.x + a0.y * b0.y;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
      const float l = lse[static_cast<size_t>(bh) * Sq + row];
      l2 = (l == kNegInf) ? __builtin_huge_valf() : l * kLog2e;
    }
    if (lane == 0) {
      lse2[r] = l2;
      dvec[r] = dsum;
    }
  }
}

// One CTA per batch row: 1 if doc[b, :] is non-decreasing.
constexpr int kSortedThreads = 256;
__global__ void __launch_bounds__(kSortedThreads)
attn_doc_sorted_kernel(const int* __restrict__ doc, int S, int* __restrict__ flags) {
  const int* d = doc + static_cast<size_t>(blockIdx.x) * S;
  int ok = 1;
  for (int i = threadIdx.x; i + 1 < S; i += kSortedThreads) ok &= (__ldg(d + i) <= __ldg(d + i + 1)) ? 1 : 0;
  ok = __syncthreads_and(ok);
  if (threadIdx.x == 0) flags[blockIdx.x] = ok;
}

// ---------------------------------------------------------------------------------------
// shared helpers
// ---------------------------------------------------------------------------------------
// First and last key (or query) position of the document run that contains position x, for
// non-decreasing ids (two binary searches).
__device__ __forceinline__ int2 doc_run(const int* drow, int S, int x) {
  const int id = __ldg(drow + x);
  int lo = 0, hi = x;
  while (lo < hi) { const int mid = (lo + hi) >> 1; if (__ldg(drow + mid) < id) lo = mid + 1; else hi = mid; }
  const int first = lo;
  lo = x + 1;
  hi = S;
  while (lo < hi) { const int mid = (lo + hi) >> 1; if (__ldg(drow + mid) <= id) lo = mid + 1; else hi = mid; }
  return make_int2(first, lo - 1);
}

// Query rows (bottom-right aligned: i' = i + Sk - Sq) that may see key j under the
// interval masks: [first, last] (unclipped).
__device__ __forceinline__ int2 rows_seeing_key(const BwdParams& p, int j) {
  const int d = p.Sk - p.Sq;
  int lo = INT_MIN / 2, hi = INT_MAX / 2;
  if (p.mask_kind & 1) lo = j - d;
  if (p.mask_kind & 2) {
    hi = j - d + p.window - 1;
    if (!(p.mask_kind & 1)) lo = j - d - p.window + 1;
  }
  return make_int2(lo, hi);
}
// Keys that query row i may see under the interval masks: [first, last] (unclipped).
__device__ __forceinline__ int2 keys_seen_by_row(const BwdParams& p, int i) {
  const int ip = i + p.Sk - p.Sq;
  int lo = 0, hi = p.Sk - 1;
  if (p.mask_kind & 1) hi = ip;
  if (p.mask_kind & 2) {
    lo = ip - p.window + 1;
    if (!(p.mask_kind & 1)) hi = ip + p.window - 1;
  }
  return make_int2(lo, hi);
}

// 128-bit mask of the visible columns clo..chi (relative to the tile, may be out of 0..127).
__device__ __forceinline__ void interval_mask(int clo, int chi, uint32_t (&vm)[4]) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int lo = min(max(clo - 32 * w, 0), 32), hi = min(max(chi + 1 - 32 * w, 0), 32);
    const uint32_t below_hi = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
    const uint32_t below_lo = lo >= 32 ? 0xffffffffu : ((1u << lo) - 1u);
    vm[w] = below_hi & ~below_lo;
  }
}

// score_mod in log2 units for one raw score s at relative position (j - i'):
// returns t and writes dt/ds / scale (1 without soft-capping) to *fp.
template <bool SOFTCAP, bool ALIBI>
__device__ __forceinline__ float bwd_modify(const BwdParams& p, float s, float slope_l2, float rel, float* fp) {
  float t;
  if constexpr (SOFTCAP) {
    const float th = tanh_approx(s * p.sc_in);
    t = th * p.sc_out;
    *fp = fmaf(-th, th, 1.f);
  } else {
    t = s * p.scale_log2;
    *fp = 1.f;
  }
  if constexpr (ALIBI) t = fmaf(slope_l2, rel, t);
  return t;
}

// Rendezvous of the 256 compute threads on an mbarrier of count 256 (one completion per use,
// `parity` the use count's low bit): arrive, then a bounded wait, so that a thread whose
// earlier wait ran out cannot leave the others waiting for ever.
__device__ __forceinline__ bool compute_sync(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             unsigned long long tmo) {
  mbar_arrive(bar);
  return __all_sync(0xffffffffu, wait_bounded(bar, parity, abort_flag, tmo));
}

// Visibility bits of 64 consecutive positions c0 .. c0+63 of a document-id row against one
// id (unsorted ids: the element test, done once per step outside the element loops).
__device__ __forceinline__ void doc_bits(const int* drow, int n, int c0, int id, uint32_t (&vm)[2]) {
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    uint32_t bits = 0u;
    for (int c = 0; c < 32; ++c) {
      const int x = c0 + 32 * w + c;
      bits |= (x < n && __ldg(drow + min(x, n - 1)) == id) ? (1u << c) : 0u;
    }
    vm[w] &= bits;
  }
}

// P (and P * dt/ds) for 64 scores of one row or column: p = 2^(t - lse), t the modified score;
// with MASKED, positions whose bit in vm is clear get p = 0.  `lse_at(e)` gives the log2 LSE
// of element e, `rel0 - sign * e` its relative position j - i'.  The loop is instantiated
// once without and once with the mask so that the common, fully visible case runs a compact,
// branch-free body.
template <bool MASKED, bool SOFTCAP, bool ALIBI, int SIGN, typename LseAt>
__device__ __forceinline__ void p_loop(const BwdParams& p, const uint32_t (&sa)[32], const uint32_t (&sb)[32],
                                       const uint32_t (&vm)[2], float slope_l2, float rel0, LseAt lse_at,
                                       uint32_t (&pk)[32], uint32_t (&pf)[32]) {
#pragma unroll
  for (int e = 0; e < 64; e += 2) {
    const float s0 = __uint_as_float(e < 32 ? sa[e] : sb[e - 32]);
    const float s1 = __uint_as_float(e + 1 < 32 ? sa[e + 1] : sb[e + 1 - 32]);
    float f0, f1;
    const float t0 = bwd_modify<SOFTCAP, ALIBI>(p, s0, slope_l2, rel0 + SIGN * e, &f0);
    const float t1 = bwd_modify<SOFTCAP, ALIBI>(p, s1, slope_l2, rel0 + SIGN * (e + 1), &f1);
    float p0 = ex2_approx(t0 - lse_at(e)), p1 = ex2_approx(t1 - lse_at(e + 1));
    if constexpr (MASKED) {
      p0 = ((vm[e >> 5] >> (e & 31)) & 1u) ? p0 : 0.f;
      p1 = ((vm[(e + 1) >> 5] >> ((e + 1) & 31)) & 1u) ? p1 : 0.f;
    }
    pk[e >> 1] = pack_bf16x2(p0, p1);
    if constexpr (SOFTCAP) pf[e >> 1] = pack_bf16x2(p0 * f0, p1 * f1);
    else pf[e >> 1] = pk[e >> 1];
  }
}

// ---------------------------------------------------------------------------------------
// dK / dV kernel
// ---------------------------------------------------------------------------------------
struct KvItem {
  int b, kvh, nt;      // batch, key/value head, key tile
  int m_lo, m_hi;      // query tiles visited: m_lo .. m_hi (per query head of the group)
  int n;               // steps = group * (m_hi - m_lo + 1), or 0
};

__device__ __forceinline__ KvItem make_kv_item(const BwdParams& p, int w) {
  KvItem it;
  const int BHkv = p.B * p.Hkv;
  int bkv;
  if (p.lpt) {   // causal: the first key tiles are seen by the most query tiles
    it.nt = w / BHkv;
    bkv = w % BHkv;
  } else {
    bkv = w / p.nkt;
    it.nt = w % p.nkt;
  }
  it.b = bkv / p.Hkv;
  it.kvh = bkv % p.Hkv;
  const int j0 = it.nt * 128, j1 = min(j0 + 127, p.Sk - 1);
  int r0 = max(rows_seeing_key(p, j0).x, 0);
  int r1 = min(rows_seeing_key(p, j1).y, p.Sq - 1);
  if (p.doc != nullptr && p.doc_sorted != nullptr && __ldg(p.doc_sorted + it.b)) {
    const int* drow = p.doc + static_cast<size_t>(it.b) * p.Sk;
    r0 = max(r0, doc_run(drow, p.Sk, j0).x);
    r1 = min(r1, doc_run(drow, p.Sk, j1).y);
  }
  if (r1 < r0) {
    it.m_lo = 0;
    it.m_hi = -1;
    it.n = 0;
    return it;
  }
  it.m_lo = r0 / 128;
  it.m_hi = r1 / 128;
  it.n = p.group * (it.m_hi - it.m_lo + 1);
  return it;
}

template <int D, bool SOFTCAP, bool ALIBI>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sptr = smem_raw + (sbase - raw);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
  // barriers: K/V of the item, the Q/dO ring, S^T and dP^T computed, P^T and dS^T written,
  // the item's last MMAs, final drain
  constexpr int B_KVFULL = 0, B_KVEMPTY = 1, B_QFULL = 2, B_QEMPTY = 2 + C::NST, B_SFULL = 2 + 2 * C::NST,
                B_DPFULL = B_SFULL + 1, B_PREADY = B_DPFULL + 1, B_DSREADY = B_PREADY + 1,
                B_DONE = B_DSREADY + 1, B_DRAIN = B_DONE + 1, B_SYNC1 = B_DRAIN + 1, B_SYNC2 = B_SYNC1 + 1;
  static_assert(B_SYNC2 < C::NBAR, "barrier count");
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sptr + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + C::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const unsigned long long tmo = p.timeout_ns;

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_KVFULL), 1);
    mbar_init(BAR(B_KVEMPTY), 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(BAR(B_QFULL + s), 1);
      mbar_init(BAR(B_QEMPTY + s), 1);
    }
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_DPFULL), 1);
    mbar_init(BAR(B_PREADY), kBwdCompute);
    mbar_init(BAR(B_DSREADY), kBwdCompute);
    mbar_init(BAR(B_DONE), 1);
    mbar_init(BAR(B_DRAIN), 1);
    mbar_init(BAR(B_SYNC1), kBwdCompute);
    mbar_init(BAR(B_SYNC2), kBwdCompute);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == kBwdLoadWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  if (warp == kBwdLoadWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_last = policy_evict_last();
      uint32_t items = 0, lidx = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int w = sched_pos(r, cta, G);
        if (w >= p.num_items) break;
        const KvItem it = make_kv_item(p, w);
        if (it.n == 0) continue;
        // K and V of this item, once the previous item's last MMAs have read them
        if (items > 0 && !wait_bounded(BAR(B_KVEMPTY), (items - 1) & 1, abort_flag, tmo)) break;
        mbar_expect_tx(BAR(B_KVFULL), 2 * C::TILE_BYTES);
        const int kvrow = it.b * p.Hkv + it.kvh;
        for (int pn = 0; pn < C::NPANEL; ++pn) {
          tma_load_3d(sbase + C::OFF_A + pn * C::PANEL_BYTES, &tm_k, BAR(B_KVFULL), pn * 64, it.nt * 128, kvrow,
                      pol_last);
          tma_load_3d(sbase + C::OFF_B + pn * C::PANEL_BYTES, &tm_v, BAR(B_KVFULL), pn * 64, it.nt * 128, kvrow,
                      pol_last);
        }
        ++items;
        const int nm = it.m_hi - it.m_lo + 1;
        for (int st = 0; st < it.n && ok; ++st) {
          const int h = it.kvh * p.group + st / nm;
          const int m = it.m_lo + st % nm;
          const uint32_t slot = lidx % C::NST;
          if (!wait_bounded(BAR(B_QEMPTY + slot), ((lidx / C::NST) & 1) ^ 1, abort_flag, tmo)) { ok = false; break; }
          const uint32_t stage = sbase + C::OFF_RING + slot * 2 * C::TILE_BYTES;
          const int bh = it.b * p.H + h;
          mbar_expect_tx(BAR(B_QFULL + slot), 2 * C::TILE_BYTES + 1024);
          for (int pn = 0; pn < C::NPANEL; ++pn) {
            tma_load_3d(stage + pn * C::PANEL_BYTES, &tm_q, BAR(B_QFULL + slot), pn * 64, m * 128, bh, pol_last);
            tma_load_3d(stage + C::TILE_BYTES + pn * C::PANEL_BYTES, &tm_do, BAR(B_QFULL + slot), pn * 64, m * 128,
                        bh, pol_last);
          }
          // LSE and Dv of the 128 rows (padded arrays: 512-byte aligned rows)
          const size_t roff = static_cast<size_t>(bh) * p.Sq_pad + static_cast<size_t>(m) * 128;
          const uint32_t rows_dst = sbase + C::OFF_ROWS + slot * 1024;
          bulk_load(rows_dst, p.lse2 + roff, 512, BAR(B_QFULL + slot));
          bulk_load(rows_dst + 512, p.dvec + roff, 512, BAR(B_QFULL + slot));
          ++lidx;
        }
      }
      // drain this thread's copies
      if (items > 0) drain_bounded(BAR(B_KVFULL), (items - 1) & 1, tmo);
      for (uint32_t idx = (lidx > C::NST ? lidx - C::NST : 0); idx < lidx; ++idx)
        drain_bounded(BAR(B_QFULL + idx % C::NST), (idx / C::NST) & 1, tmo);
    }
  } else if (warp == kBwdMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS = tbase + C::T_S, tDP = tbase + C::T_DP, tDV = tbase + C::T_ACC0, tDK = tbase + C::T_ACC1;
      const uint64_t dk_k = make_sdesc_sw128(sbase + C::OFF_A, 16, 1024);       // K as K-major A
      const uint64_t dv_k = make_sdesc_sw128(sbase + C::OFF_B, 16, 1024);       // V as K-major A
      const uint64_t dring_k = make_sdesc_sw128(sbase + C::OFF_RING, 16, 1024);           // K-major B
      const uint64_t dring_mn = make_sdesc_sw128(sbase + C::OFF_RING, C::PANEL_BYTES, 1024);  // MN-major B
      auto ss = [&](uint32_t dst, uint64_t a0, uint64_t b0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int col = kk * 16;
          const uint32_t off = ((col / 64) * C::PANEL_BYTES + (col % 64) * 2) >> 4;
          mma_f16_ss(dst, a0 + off, b0 + off, C::IDESC_SS, kk > 0);
        }
      };
      auto ts = [&](uint32_t dst, uint32_t a_tmem, uint64_t b0, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ts(dst, a_tmem + kk * 8, b0 + ((kk * 16 * 128) >> 4), C::IDESC_TS, (acc || kk > 0) ? 1u : 0u);
      };
      auto soff = [&](uint32_t idx) -> uint32_t { return ((idx % C::NST) * 2 * C::TILE_BYTES) >> 4; };
      uint32_t items = 0, cidx = 0, tcount = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int w = sched_pos(r, cta, G);
        if (w >= p.num_items) break;
        const KvItem it = make_kv_item(p, w);
        if (it.n == 0) continue;
        if (!wait_bounded(BAR(B_KVFULL), items & 1, abort_flag, tmo)) { ok = false; break; }
        if (!wait_bounded(BAR(B_QFULL + cidx % C::NST), (cidx / C::NST) & 1, abort_flag, tmo)) { ok = false; break; }
        tc_fence_after();
        // step 0: S^T = K Q^T and dP^T = V dO^T
        ss(tS, dk_k, dring_k + soff(cidx));
        mma_commit(BAR(B_SFULL));
        ss(tDP, dv_k, dring_k + soff(cidx) + (C::TILE_BYTES >> 4));
        mma_commit(BAR(B_DPFULL));
        for (int st = 0; st < it.n; ++st) {
          const uint32_t idx = cidx + st, t = tcount + st;
          const bool more = st + 1 < it.n;
          // dV += P^T dO once P^T is written; then the next S^T (over P^T: this thread's
          // MMAs execute in issue order, so dV reads P^T first)
          if (!wait_bounded(BAR(B_PREADY), t & 1, abort_flag, tmo)) { ok = false; break; }
          tc_fence_after();
          ts(tDV, tS, dring_mn + soff(idx) + (C::TILE_BYTES >> 4), st > 0);
          if (more) {
            if (!wait_bounded(BAR(B_QFULL + (idx + 1) % C::NST), ((idx + 1) / C::NST) & 1, abort_flag, tmo)) {
              ok = false;
              break;
            }
            tc_fence_after();
            ss(tS, dk_k, dring_k + soff(idx + 1));
            mma_commit(BAR(B_SFULL));
          }
          // dK += dS^T Q once dS^T is written; then the stage is free and the next dP^T
          if (!wait_bounded(BAR(B_DSREADY), t & 1, abort_flag, tmo)) { ok = false; break; }
          tc_fence_after();
          ts(tDK, tDP, dring_mn + soff(idx), st > 0);
          mma_commit(BAR(B_QEMPTY + idx % C::NST));
          if (more) {
            ss(tDP, dv_k, dring_k + soff(idx + 1) + (C::TILE_BYTES >> 4));
            mma_commit(BAR(B_DPFULL));
          }
        }
        if (!ok) break;
        mma_commit(BAR(B_KVEMPTY));
        mma_commit(BAR(B_DONE));
        cidx += it.n;
        tcount += it.n;
        ++items;
      }
      mma_commit(BAR(B_DRAIN));
      drain_bounded(BAR(B_DRAIN), 0, tmo);
    }
  } else {
    // ------------------------------------------------------------------ compute warps
    const int quarter = warp & 3, half = warp >> 2;
    const int rloc = quarter * 32 + lane;                    // key row within the tile (TMEM lane)
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tbase + C::T_S + lane_off, tDP = tbase + C::T_DP + lane_off;
    const int col0 = 64 * half;                              // this warp's query columns col0 .. col0+63
    const float* srows = reinterpret_cast<const float*>(sptr + C::OFF_ROWS);
    uint32_t tcount = 0, cidx = 0, items = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int w = sched_pos(r, cta, G);
      if (w >= p.num_items) break;
      const KvItem it = make_kv_item(p, w);
      const int j = it.nt * 128 + rloc;                      // key position
      if (it.n == 0) {
        // no query row sees this key tile: dK = dV = 0 (warps 0-3 write dV, 4-7 dK)
        if (j < p.Sk) {
          __nv_bfloat16* dst = (half == 0 ? p.dv : p.dk) + (static_cast<size_t>(it.b * p.Hkv + it.kvh) * p.Sk + j) * D;
          for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(dst + c) = make_uint4(0u, 0u, 0u, 0u);
        }
        continue;
      }
      const int2 rs = rows_seeing_key(p, j);
      int ilo = rs.x, ihi = min(rs.y, p.Sq - 1);
      if (j >= p.Sk) ihi = -1;                               // padding key: sees nothing
      const bool has_doc = p.doc != nullptr;
      bool doc_elem = false;
      int doc_j = 0;
      const int* drow = has_doc ? p.doc + static_cast<size_t>(it.b) * p.Sk : nullptr;
      if (has_doc && j < p.Sk) {
        if (p.doc_sorted != nullptr && __ldg(p.doc_sorted + it.b)) {
          const int2 run = doc_run(drow, p.Sk, j);
          ilo = max(ilo, run.x);
          ihi = min(ihi, run.y);
        } else {
          doc_elem = true;
          doc_j = __ldg(drow + j);
        }
      }
      const int nm = it.m_hi - it.m_lo + 1;
      const int d = p.Sk - p.Sq;
      for (int st = 0; st < it.n; ++st) {
        const int h = it.kvh * p.group + st / nm;
        const int m = it.m_lo + st % nm;
        const uint32_t slot = (cidx + st) % C::NST;
        const uint32_t t = tcount + st;
        float slope_l2 = 0.f;
        if constexpr (ALIBI) slope_l2 = __ldg(p.alibi + h) * kLog2e;
        // the stage's rows of LSE and Dv came by bulk copy: observe that copy's barrier too
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(B_QFULL + slot), ((cidx + st) / C::NST) & 1, abort_flag, tmo) &&
                                     wait_bounded(BAR(B_SFULL), t & 1, abort_flag, tmo))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* lse_row = srows + slot * 256 + col0;
        const float4* dvv4 = reinterpret_cast<const float4*>(srows + slot * 256 + 128 + col0);
        // every query column of this warp's half visible to this key row (and no element test)
        const int q0 = m * 128 + col0;
        const bool full = __all_sync(0xffffffffu, !doc_elem && ilo <= q0 && ihi >= q0 + 63);
        uint32_t vm[2] = {0xffffffffu, 0xffffffffu};
        if (!full) {
          uint32_t v4[4];
          interval_mask(ilo - m * 128, ihi - m * 128, v4);
          vm[0] = half ? v4[2] : v4[0];
          vm[1] = half ? v4[3] : v4[1];
          if (doc_elem) doc_bits(drow, p.Sq, q0, doc_j, vm);
        }
        const float rel0 = static_cast<float>(j - d - q0);         // j - i' for this warp's column 0
        // ---- pass 1: P^T = exp2(t - lse2), kept in registers as P * dt/ds for pass 2
        uint32_t sa[32], sb[32];
        tmem_ld_x32_wait(tS + col0, sa);
        tmem_ld_x32_wait(tS + col0 + 32, sb);
        // every warp has read its S^T columns before any P^T is written over them
        if (!compute_sync(BAR(B_SYNC1), t & 1, abort_flag, tmo)) { ok = false; break; }
        uint32_t pk[32], pf[32];
        auto lse_at = [&](int e) -> float { return lse_row[e]; };
        if (full) p_loop<false, SOFTCAP, ALIBI, -1>(p, sa, sb, vm, slope_l2, rel0, lse_at, pk, pf);
        else p_loop<true, SOFTCAP, ALIBI, -1>(p, sa, sb, vm, slope_l2, rel0, lse_at, pk, pf);
        tmem_st_x32_wait<0>(tS + (col0 >> 1), pk);   // P^T: query pair (2c, 2c+1) in column c
        tc_fence_before();
        mbar_arrive(BAR(B_PREADY));
        // ---- pass 2: dS^T = (P dt/ds) (dP^T - Dv) over dP^T's first 64 columns
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(B_DPFULL), t & 1, abort_flag, tmo))) { ok = false; break; }
        tc_fence_after();
        tmem_ld_x32_wait(tDP + col0, sa);
        tmem_ld_x32_wait(tDP + col0 + 32, sb);
        // every warp has read its dP^T columns before any dS^T is written over them
        if (!compute_sync(BAR(B_SYNC2), t & 1, abort_flag, tmo)) { ok = false; break; }
        uint32_t dk[32];
#pragma unroll
        for (int e4 = 0; e4 < 16; ++e4) {
          const float4 d4 = dvv4[e4];
          const float dl[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int u = 0; u < 4; u += 2) {
            const int e = 4 * e4 + u;
            const float2 pp = unpack_bf16x2(pf[e >> 1]);
            const float x0 = __uint_as_float(e < 32 ? sa[e] : sb[e - 32]);
            const float x1 = __uint_as_float(e + 1 < 32 ? sa[e + 1] : sb[e + 1 - 32]);
            dk[e >> 1] = pack_bf16x2(pp.x * (x0 - dl[u]), pp.y * (x1 - dl[u + 1]));
          }
        }
        tmem_st_x32_wait<0>(tDP + (col0 >> 1), dk);
        tc_fence_before();
        mbar_arrive(BAR(B_DSREADY));
      }
      if (!__all_sync(0xffffffffu, ok && !*abort_flag)) {
        ok = false;
        break;
      }
      // ---- epilogue: warps 0-3 write dV, warps 4-7 write scale * dK (bf16)
      if (!__all_sync(0xffffffffu, wait_bounded(BAR(B_DONE), items & 1, abort_flag, tmo))) { ok = false; break; }
      tc_fence_after();
      {
        const size_t orow = (static_cast<size_t>(it.b * p.Hkv + it.kvh) * p.Sk + j) * D;
        __nv_bfloat16* dst = (half == 0 ? p.dv : p.dk) + orow;
        const float mul = half == 0 ? 1.f : p.scale;
        const uint32_t src = tbase + (half == 0 ? C::T_ACC0 : C::T_ACC1) + lane_off;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t a[32];
          tmem_ld_x32_wait(src + ch * 32, a);
          uint32_t wv[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            wv[c] = pack_bf16x2(__uint_as_float(a[2 * c]) * mul, __uint_as_float(a[2 * c + 1]) * mul);
          if (j < p.Sk) {
            uint4* o4 = reinterpret_cast<uint4*>(dst + ch * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) o4[v] = make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]);
          }
        }
      }
      tc_fence_before();
      cidx += it.n;
      tcount += it.n;
      ++items;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------
// dQ kernel
// ---------------------------------------------------------------------------------------
struct QItem {
  int b, h, bh, mt;    // batch, head, b*H+h, query tile
  int kt_lo, n;        // key tiles kt_lo .. kt_lo + n - 1
};

__device__ __forceinline__ QItem make_q_item(const BwdParams& p, int w) {
  QItem it;
  const int BH = p.B * p.H;
  if (p.lpt) {   // causal: the last query tiles see the most key tiles
    it.mt = p.nqt - 1 - w / BH;
    it.bh = w % BH;
  } else {
    it.bh = w / p.nqt;
    it.mt = w % p.nqt;
  }
  it.b = it.bh / p.H;
  it.h = it.bh % p.H;
  const int i0 = it.mt * 128, i1 = min(i0 + 127, p.Sq - 1);
  int c0 = max(keys_seen_by_row(p, i0).x, 0);
  int c1 = min(keys_seen_by_row(p, i1).y, p.Sk - 1);
  if (p.doc != nullptr && p.doc_sorted != nullptr && __ldg(p.doc_sorted + it.b)) {
    const int* drow = p.doc + static_cast<size_t>(it.b) * p.Sk;
    c0 = max(c0, doc_run(drow, p.Sk, i0).x);
    c1 = min(c1, doc_run(drow, p.Sk, i1).y);
  }
  if (c1 < c0) {
    it.kt_lo = 0;
    it.n = 0;
    return it;
  }
  it.kt_lo = c0 / 128;
  it.n = c1 / 128 - it.kt_lo + 1;
  return it;
}

template <int D, bool SOFTCAP, bool ALIBI>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sptr = smem_raw + (sbase - raw);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::DQ_OFF_BAR + 8 * i; };
  // barriers: Q/dO of the item, the K ring, the V ring, S computed, S read by the compute
  // warps, dP computed (one per dP buffer), dS written, the item's last MMA, final drain,
  // compute rendezvous
  constexpr int NK = C::DQ_NK, NV = C::DQ_NV;
  constexpr int B_QFULL = 0, B_QEMPTY = 1, B_KFULL = 2, B_KEMPTY = 2 + NK, B_VFULL = 2 + 2 * NK,
                B_VEMPTY = B_VFULL + NV, B_SFULL = B_VEMPTY + NV, B_SFREE = B_SFULL + 1, B_DPFULL = B_SFREE + 1,
                B_DSREADY = B_DPFULL + 2, B_DONE = B_DSREADY + 1, B_DRAIN = B_DONE + 1, B_SYNC = B_DRAIN + 1;
  static_assert(B_SYNC < C::NBAR, "barrier count");
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sptr + C::DQ_OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + C::DQ_OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const unsigned long long tmo = p.timeout_ns;

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_QFULL), 1);
    mbar_init(BAR(B_QEMPTY), 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(BAR(B_KFULL + s), 1);
      mbar_init(BAR(B_KEMPTY + s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(BAR(B_VFULL + s), 1);
      mbar_init(BAR(B_VEMPTY + s), 1);
    }
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_SFREE), kBwdCompute);
    mbar_init(BAR(B_DPFULL), 1);
    mbar_init(BAR(B_DPFULL + 1), 1);
    mbar_init(BAR(B_DSREADY), kBwdCompute);
    mbar_init(BAR(B_DONE), 1);
    mbar_init(BAR(B_DRAIN), 1);
    mbar_init(BAR(B_SYNC), kBwdCompute);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == kBwdLoadWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  if (warp == kBwdLoadWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_last = policy_evict_last();
      const uint64_t pol_first = policy_evict_first();
      uint32_t items = 0, lidx = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int w = sched_pos(r, cta, G);
        if (w >= p.num_items) break;
        const QItem it = make_q_item(p, w);
        if (it.n == 0) continue;
        if (items > 0 && !wait_bounded(BAR(B_QEMPTY), (items - 1) & 1, abort_flag, tmo)) break;
        mbar_expect_tx(BAR(B_QFULL), 2 * C::TILE_BYTES);
        for (int pn = 0; pn < C::NPANEL; ++pn) {
          tma_load_3d(sbase + C::OFF_A + pn * C::PANEL_BYTES, &tm_q, BAR(B_QFULL), pn * 64, it.mt * 128, it.bh,
                      pol_first);
          tma_load_3d(sbase + C::OFF_B + pn * C::PANEL_BYTES, &tm_do, BAR(B_QFULL), pn * 64, it.mt * 128, it.bh,
                      pol_first);
        }
        ++items;
        const int kvrow = it.b * p.Hkv + it.h / p.group;
        for (int st = 0; st < it.n && ok; ++st) {
          const int kt = it.kt_lo + st;
          // K and V of step lidx, each into its own ring
          const uint32_t ks = lidx % NK, vs = lidx % NV;
          if (!wait_bounded(BAR(B_KEMPTY + ks), ((lidx / NK) & 1) ^ 1, abort_flag, tmo)) { ok = false; break; }
          mbar_expect_tx(BAR(B_KFULL + ks), C::TILE_BYTES);
          for (int pn = 0; pn < C::NPANEL; ++pn)
            tma_load_3d(sbase + C::DQ_OFF_K + ks * C::TILE_BYTES + pn * C::PANEL_BYTES, &tm_k, BAR(B_KFULL + ks),
                        pn * 64, kt * 128, kvrow, pol_last);
          if (!wait_bounded(BAR(B_VEMPTY + vs), ((lidx / NV) & 1) ^ 1, abort_flag, tmo)) { ok = false; break; }
          mbar_expect_tx(BAR(B_VFULL + vs), C::TILE_BYTES);
          for (int pn = 0; pn < C::NPANEL; ++pn)
            tma_load_3d(sbase + C::DQ_OFF_V + vs * C::TILE_BYTES + pn * C::PANEL_BYTES, &tm_v, BAR(B_VFULL + vs),
                        pn * 64, kt * 128, kvrow, pol_last);
          ++lidx;
        }
      }
      if (items > 0) drain_bounded(BAR(B_QFULL), (items - 1) & 1, tmo);
      for (uint32_t idx = (lidx > NK ? lidx - NK : 0); idx < lidx; ++idx)
        drain_bounded(BAR(B_KFULL + idx % NK), (idx / NK) & 1, tmo);
      for (uint32_t idx = (lidx > NV ? lidx - NV : 0); idx < lidx; ++idx)
        drain_bounded(BAR(B_VFULL + idx % NV), (idx / NV) & 1, tmo);
    }
  } else if (warp == kBwdMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS = tbase + C::T_S, tDQ = tbase + C::T_DQ;
      auto tDPb = [&](uint32_t t) -> uint32_t { return tbase + ((t & 1u) ? C::T_DP1 : C::T_DP0); };
      const uint64_t dq_k = make_sdesc_sw128(sbase + C::OFF_A, 16, 1024);
      const uint64_t ddo_k = make_sdesc_sw128(sbase + C::OFF_B, 16, 1024);
      const uint64_t dk_k = make_sdesc_sw128(sbase + C::DQ_OFF_K, 16, 1024);                  // K, K-major (S)
      const uint64_t dk_mn = make_sdesc_sw128(sbase + C::DQ_OFF_K, C::PANEL_BYTES, 1024);     // K, MN-major (dQ)
      const uint64_t dv_k = make_sdesc_sw128(sbase + C::DQ_OFF_V, 16, 1024);                  // V, K-major (dP)
      auto ss = [&](uint32_t dst, uint64_t a0, uint64_t b0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int col = kk * 16;
          const uint32_t off = ((col / 64) * C::PANEL_BYTES + (col % 64) * 2) >> 4;
          mma_f16_ss(dst, a0 + off, b0 + off, C::IDESC_SS, kk > 0);
        }
      };
      auto koff = [&](uint32_t idx) -> uint32_t { return ((idx % NK) * C::TILE_BYTES) >> 4; };
      auto voff = [&](uint32_t idx) -> uint32_t { return ((idx % NV) * C::TILE_BYTES) >> 4; };
      auto k_ready = [&](uint32_t idx) -> bool {
        return wait_bounded(BAR(B_KFULL + idx % NK), (idx / NK) & 1, abort_flag, tmo);
      };
      auto v_ready = [&](uint32_t idx) -> bool {
        return wait_bounded(BAR(B_VFULL + idx % NV), (idx / NV) & 1, abort_flag, tmo);
      };
      // dP of step index idx into dP buffer t & 1; its V slot is free once the MMA is done
      auto dp_step = [&](uint32_t idx, uint32_t t) -> bool {
        if (!v_ready(idx)) return false;
        tc_fence_after();
        ss(tDPb(t), ddo_k, dv_k + voff(idx));
        mma_commit(BAR(B_DPFULL + (t & 1)));
        mma_commit(BAR(B_VEMPTY + idx % NV));
        return true;
      };
      uint32_t items = 0, cidx = 0, tcount = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int w = sched_pos(r, cta, G);
        if (w >= p.num_items) break;
        const QItem it = make_q_item(p, w);
        if (it.n == 0) continue;
        if (!wait_bounded(BAR(B_QFULL), items & 1, abort_flag, tmo) || !k_ready(cidx)) { ok = false; break; }
        tc_fence_after();
        // S(0) = Q K^T, dP(0) = dO V^T, and dP(1) ahead into the other dP buffer
        ss(tS, dq_k, dk_k + koff(cidx));
        mma_commit(BAR(B_SFULL));
        if (!dp_step(cidx, tcount) || (it.n > 1 && !dp_step(cidx + 1, tcount + 1))) { ok = false; break; }
        for (int st = 0; st < it.n; ++st) {
          const uint32_t idx = cidx + st, t = tcount + st;
          // S of the next step once the compute warps have read this one
          if (!wait_bounded(BAR(B_SFREE), t & 1, abort_flag, tmo)) { ok = false; break; }
          if (st + 1 < it.n) {
            if (!k_ready(idx + 1)) { ok = false; break; }
            tc_fence_after();
            ss(tS, dq_k, dk_k + koff(idx + 1));
            mma_commit(BAR(B_SFULL));
          }
          // dQ += dS K once dS is written (over this step's dP); then K of this step is free
          if (!wait_bounded(BAR(B_DSREADY), t & 1, abort_flag, tmo)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16_ts(tDQ, tDPb(t) + kk * 8, dk_mn + koff(idx) + ((kk * 16 * 128) >> 4), C::IDESC_TS,
                       (st > 0 || kk > 0) ? 1u : 0u);
          mma_commit(BAR(B_KEMPTY + idx % NK));
          // dP two steps ahead, into the buffer dQ has just read
          if (st + 2 < it.n && !dp_step(idx + 2, t)) { ok = false; break; }
        }
        if (!ok) break;
        mma_commit(BAR(B_QEMPTY));
        mma_commit(BAR(B_DONE));
        cidx += it.n;
        tcount += it.n;
        ++items;
      }
      mma_commit(BAR(B_DRAIN));
      drain_bounded(BAR(B_DRAIN), 0, tmo);
    }
  } else {
    // ------------------------------------------------------------------ compute warps
    const int quarter = warp & 3, half = warp >> 2;
    const int rloc = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tbase + C::T_S + lane_off;
    const int col0 = 64 * half;                              // this warp's key columns col0 .. col0+63
    uint32_t tcount = 0, items = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int w = sched_pos(r, cta, G);
      if (w >= p.num_items) break;
      const QItem it = make_q_item(p, w);
      const int i = it.mt * 128 + rloc;
      if (it.n == 0) {
        // rows that see no key: dQ = 0 (each half writes half of the row)
        if (i < p.Sq) {
          __nv_bfloat16* dst = p.dq + (static_cast<size_t>(it.bh) * p.Sq + i) * D + half * (D / 2);
          for (int c = 0; c < D / 2; c += 8) *reinterpret_cast<uint4*>(dst + c) = make_uint4(0u, 0u, 0u, 0u);
        }
        continue;
      }
      const int2 ks = keys_seen_by_row(p, i);
      int jlo = ks.x, jhi = min(ks.y, p.Sk - 1);
      if (i >= p.Sq) jhi = -1;
      const bool has_doc = p.doc != nullptr;
      bool doc_elem = false;
      int doc_i = 0;
      const int* drow = has_doc ? p.doc + static_cast<size_t>(it.b) * p.Sk : nullptr;
      if (has_doc && i < p.Sq) {
        if (p.doc_sorted != nullptr && __ldg(p.doc_sorted + it.b)) {
          const int2 run = doc_run(drow, p.Sk, i);
          jlo = max(jlo, run.x);
          jhi = min(jhi, run.y);
        } else {
          doc_elem = true;
          doc_i = __ldg(drow + i);
        }
      }
      const size_t rr = static_cast<size_t>(it.bh) * p.Sq_pad + i;
      const float lse2 = __ldg(p.lse2 + rr);
      const float dvi = __ldg(p.dvec + rr);
      float slope_l2 = 0.f;
      if constexpr (ALIBI) slope_l2 = __ldg(p.alibi + it.h) * kLog2e;
      const int ip = i + p.Sk - p.Sq;
      for (int st = 0; st < it.n; ++st) {
        const uint32_t t = tcount + st;
        const int kt = it.kt_lo + st;
        const uint32_t tDP = tbase + ((t & 1u) ? C::T_DP1 : C::T_DP0) + lane_off;
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(B_SFULL), t & 1, abort_flag, tmo))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int c0 = kt * 128 + col0;
        const bool full = __all_sync(0xffffffffu, !doc_elem && jlo <= c0 && jhi >= c0 + 63);
        uint32_t vm[2] = {0xffffffffu, 0xffffffffu};
        if (!full) {
          uint32_t v4[4];
          interval_mask(jlo - kt * 128, jhi - kt * 128, v4);
          vm[0] = half ? v4[2] : v4[0];
          vm[1] = half ? v4[3] : v4[1];
          if (doc_elem) doc_bits(drow, p.Sk, c0, doc_i, vm);
        }
        const float rel0 = static_cast<float>(c0 - ip);      // j - i' for this warp's column 0
        uint32_t sa[32], sb[32];
        tmem_ld_x32_wait(tS + col0, sa);
        tmem_ld_x32_wait(tS + col0 + 32, sb);
        // S is in registers: the MMA may compute the next step's S over it
        tc_fence_before();
        mbar_arrive(BAR(B_SFREE));
        // P * dt/ds rounded to bf16 first, as in the dK/dV kernel, so that both use the same dS
        uint32_t pk[32], pf[32];
        auto lse_at = [&](int) -> float { return lse2; };
        if (full) p_loop<false, SOFTCAP, ALIBI, 1>(p, sa, sb, vm, slope_l2, rel0, lse_at, pk, pf);
        else p_loop<true, SOFTCAP, ALIBI, 1>(p, sa, sb, vm, slope_l2, rel0, lse_at, pk, pf);
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(B_DPFULL + (t & 1)), (t >> 1) & 1, abort_flag, tmo))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t da[32], db[32];
        tmem_ld_x32_wait(tDP + col0, da);
        tmem_ld_x32_wait(tDP + col0 + 32, db);
        // every warp has read its dP columns before any dS is written over them
        if (!compute_sync(BAR(B_SYNC), t & 1, abort_flag, tmo)) { ok = false; break; }
        uint32_t dk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const float2 pp = unpack_bf16x2(pf[e >> 1]);
          const float x0 = __uint_as_float(e < 32 ? da[e] : db[e - 32]);
          const float x1 = __uint_as_float(e + 1 < 32 ? da[e + 1] : db[e + 1 - 32]);
          dk[e >> 1] = pack_bf16x2(pp.x * (x0 - dvi), pp.y * (x1 - dvi));
        }
        tmem_st_x32_wait<0>(tDP + (col0 >> 1), dk);   // dS: key pair (2c, 2c+1) in column c
        tc_fence_before();
        mbar_arrive(BAR(B_DSREADY));
      }
      if (!__all_sync(0xffffffffu, ok && !*abort_flag)) {
        ok = false;
        break;
      }
      if (!__all_sync(0xffffffffu, wait_bounded(BAR(B_DONE), items & 1, abort_flag, tmo))) { ok = false; break; }
      tc_fence_after();
      // each half of the warps writes half of the dQ row (scale * dQ, bf16)
      __nv_bfloat16* dst = p.dq + (static_cast<size_t>(it.bh) * p.Sq + i) * D;
      const uint32_t src = tbase + C::T_DQ + lane_off;
#pragma unroll
      for (int ch = 0; ch < D / 64; ++ch) {
        const int cc = half * (D / 2) + ch * 32;
        uint32_t a[32];
        tmem_ld_x32_wait(src + cc, a);
        uint32_t wv[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          wv[c] = pack_bf16x2(__uint_as_float(a[2 * c]) * p.scale, __uint_as_float(a[2 * c + 1]) * p.scale);
        if (i < p.Sq) {
          uint4* o4 = reinterpret_cast<uint4*>(dst + cc);
#pragma unroll
          for (int v = 0; v < 4; ++v) o4[v] = make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]);
        }
      }
      tc_fence_before();
      tcount += it.n;
      ++items;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace attn
