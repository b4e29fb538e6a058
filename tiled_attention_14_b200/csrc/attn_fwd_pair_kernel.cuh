// attn_fwd_pair_kernel.cuh — the BF16 attention forward (D = 128) on pairs of SMs.
//
// Same computation, work items and masks as attn_fwd_kernel (one (b, h) and one block of
// 256 query rows per item; the 256x128 Blackwell tile of the FlexAttention page, section
// "Aktuelle Einschränkungen"), but each item runs on a cluster of two CTAs on two SMs:
//   - the pair MMA (tcgen05 cta_group::2, M = 256) computes S = Q K^T and O += P V for all 256
//     rows; CTA r keeps rows 128r .. 128r+127 of S, P and O in its own tensor memory;
//   - each CTA loads its own 128 query rows and HALF of every K/V tile (K: keys 64r .. 64r+63
//     of the tile, V: value columns 64r .. 64r+63), so an SM streams half the K/V bytes of the
//     single-CTA kernel per 128 rows;
//   - tensor memory per SM then has room for two S buffers and O (S_a | S_b | O): S of the
//     next key tile is computed while the softmax warps work on this one, so the softmax runs
//     back to back instead of waiting for P V and the next S of the same rows (the chain that
//     bounds the single-CTA kernel, where P aliases the only S buffer of each query tile);
//   - eight softmax warps per CTA, two per TMEM lane quarter: each thread owns one query row and
//     one half (64 keys) of every key tile; the two halves of a row combine their maxima once
//     per tile through shared memory (a bounded mbarrier rendezvous) and their sums at the end.
// The on-chip storage limit that the FP4 FlashAttention-4 page names (tensor memory too full
// to overlap stages, paragraph on on-chip storage) is what the pair split relieves.
//
// Roles (384 threads per CTA): warps 0-7 softmax, warp 8 TMA producer (each CTA loads its own
// halves; the byte counts of both land on the even CTA's barriers), warp 9 MMA issuer (even
// CTA only; it also allocates the pair's tensor memory with its peer warp), warps 10-11 idle.
// Every wait is bounded; no TMA multicast.  Both CTAs meet at a cluster barrier after setup and
// before tensor memory is freed, and every path (time-outs included) reaches it.  Hand-offs
// between the CTAs use CTA-scope release / acquire: nothing in generic memory crosses the
// pair (tensor memory and the TMA / MMA transactions are ordered by the tcgen05 fences and
// the barriers' transaction counts), and cluster-scope semantics cost about 550 clocks per
// hand-off (measured on B200).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "attn_fwd_kernel.cuh"

namespace attn {

template <int NSPLIT>
struct CfgPair {
  // NSPLIT softmax warps per TMEM lane quarter; each takes 128 / NSPLIT keys of every tile
  static_assert(NSPLIT == 2 || NSPLIT == 4, "column split");
  static constexpr int THREADS = 128 * (NSPLIT + 1);   // softmax warpgroups + one control warpgroup
  static constexpr int LOAD_WARP = 4 * NSPLIT, MMA_WARP = 4 * NSPLIT + 1;
  static constexpr int COLS = 128 / NSPLIT;
  static constexpr int D = 128;
  static constexpr int Q_BYTES = 128 * D * 2;          // this CTA's 128 query rows (two 64-column panels)
  static constexpr int QPANEL = 128 * 128;             // 128 rows x 128 bytes
  static constexpr int HALF = 16384;                   // K half (64 keys) or V half (64 columns) of a tile
  static constexpr int STAGE = 2 * HALF;               // ring stage: this CTA's K half at +0, V half at +HALF
  static constexpr int KPANEL = 64 * 128;              // K half: 64 keys x 128 bytes per 64-column panel
  static constexpr int NS = 4;                         // ring depth in key tiles
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = Q_BYTES;
  static constexpr int OFF_XCH = OFF_KV + NS * STAGE;  // [2 slots][NSPLIT parts][128 rows] floats
  static constexpr int XCH_BYTES = 2 * NSPLIT * 128 * 4;
  static constexpr int OFF_BAR = OFF_XCH + XCH_BYTES;
  // q_full, q_empty, kv_full[NS], kv_empty[NS], s_full[2], p_full[2], o_done, drain, xch[4]
  static constexpr int B_QFULL = 0, B_QEMPTY = 1, B_KVFULL = 2, B_KVEMPTY = 2 + NS, B_SFULL = 2 + 2 * NS,
                       B_PFULL = B_SFULL + 2, B_ODONE = B_PFULL + 2, B_DRAIN = B_ODONE + 1, B_XCH = B_DRAIN + 1;
  static constexpr int NBAR = B_XCH + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base (4 B), abort flag (4 B)
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S0 = 0, T_S1 = 128, T_O = 256;
  static constexpr uint32_t IDESC_QK = make_idesc(1u, 256, 128, false);
  static constexpr uint32_t IDESC_PV = make_idesc(1u, 256, D, true);
  static constexpr int P_ARRIVALS = 2 * 4 * NSPLIT;    // p_full: one per softmax warp of both CTAs
};

// One key tile of the online softmax for one part (128 / NSPLIT keys) of one query row: reads
// the part's scores, applies score_mod and the mask, combines the row maximum with the other
// parts, updates the running maximum (rescale threshold as in the single-CTA kernel), writes P
// (bf16, key pair 2c, 2c+1 in column c of the part's columns) over the S buffer and rescales
// the part's columns of O when the maximum moved, once P V of the previous key
// tile is known complete (phase prev_par of prev_bar, unless *prev_done).  Returns false on
// time-out.
template <int NSPLIT, bool SOFTCAP, bool ALIBI>
__device__ __forceinline__ bool softmax_part(const FwdParams& p, const Item& it, int kt, int cls, int part,
                                             int rloc, uint32_t tS, uint32_t tO, int ip, int jlo_row, int jhi_row,
                                             bool doc_elem, int doc_row, float slope_l2, float* xch,
                                             uint32_t xbar, uint32_t& xc, uint32_t prev_bar, uint32_t prev_par,
                                             bool* prev_done, uint32_t t, volatile int* abort_flag, unsigned long long tmo, float& m_run,
                                             float& l_part) {
  constexpr int COLS = 128 / NSPLIT;
  const int col0 = COLS * part;
  uint32_t s[COLS];
  if constexpr (COLS == 64) tmem_ld_x64_wait(tS + col0, s);
  else tmem_ld_x32_wait(tS + col0, s);
  const float sc = p.scale_log2;
  const int c0 = kt * 128 + col0;                      // key of column 0 of this part
  constexpr bool kPlain = !SOFTCAP && !ALIBI;
  float alibi_base = 0.f;
  if constexpr (ALIBI) alibi_base = slope_l2 * static_cast<float>(c0 - ip);
  auto modify = [&](float v, int c) -> float {
    if constexpr (!kPlain) {
      if constexpr (SOFTCAP) {
        v = tanh_approx(v * p.sc_in) * p.sc_out;
        if constexpr (ALIBI) v = fmaf(slope_l2, static_cast<float>(c), v + alibi_base);
      } else if constexpr (ALIBI) {
        v = fmaf(v, sc, fmaf(slope_l2, static_cast<float>(c), alibi_base));
      }
    }
    return v;
  };
  float mxa[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) mxa[u] = kNegInf;
  const bool masked = (cls == 1);
  if (masked) {
    const int clo = jlo_row - c0, chi = jhi_row - c0;
    if (!doc_elem) {
      uint32_t vm[COLS / 32];
#pragma unroll
      for (int w = 0; w < COLS / 32; ++w) {
        const int lo = min(max(clo - 32 * w, 0), 32), hi = min(max(chi + 1 - 32 * w, 0), 32);
        const uint32_t below_hi = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
        const uint32_t below_lo = lo >= 32 ? 0xffffffffu : ((1u << lo) - 1u);
        vm[w] = below_hi & ~below_lo;
      }
      auto visible = [&](int c) -> bool {
        if constexpr (ALIBI) return c >= clo && c <= chi;
        else return ((vm[c >> 5] >> (c & 31)) & 1u) != 0u;
      };
#pragma unroll
      for (int c = 0; c < COLS; c += 2) {
        float t0 = modify(__uint_as_float(s[c]), c);
        float t1 = modify(__uint_as_float(s[c + 1]), c + 1);
        t0 = visible(c) ? t0 : kNegInf;
        t1 = visible(c + 1) ? t1 : kNegInf;
        s[c] = __float_as_uint(t0);
        s[c + 1] = __float_as_uint(t1);
        mxa[(c >> 1) & 7] = fmax3f(mxa[(c >> 1) & 7], t0, t1);
      }
    } else {
      // unsorted document ids: element test against the row's id (key index clamped into the row)
      const int* drow = p.doc + static_cast<size_t>(it.b) * p.Sk;
      const int last = p.Sk - 1;
#pragma unroll
      for (int c = 0; c < COLS; c += 2) {
        float t0 = modify(__uint_as_float(s[c]), c);
        float t1 = modify(__uint_as_float(s[c + 1]), c + 1);
        const bool v0 = c >= clo && c <= chi && c0 + c <= last && __ldg(drow + min(c0 + c, last)) == doc_row;
        const bool v1 =
            c + 1 >= clo && c + 1 <= chi && c0 + c + 1 <= last && __ldg(drow + min(c0 + c + 1, last)) == doc_row;
        t0 = v0 ? t0 : kNegInf;
        t1 = v1 ? t1 : kNegInf;
        s[c] = __float_as_uint(t0);
        s[c + 1] = __float_as_uint(t1);
        mxa[(c >> 1) & 7] = fmax3f(mxa[(c >> 1) & 7], t0, t1);
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < COLS; c += 2) {
      const float t0 = modify(__uint_as_float(s[c]), c);
      const float t1 = modify(__uint_as_float(s[c + 1]), c + 1);
      if constexpr (!kPlain) {
        s[c] = __float_as_uint(t0);
        s[c + 1] = __float_as_uint(t1);
      }
      mxa[(c >> 1) & 7] = fmax3f(mxa[(c >> 1) & 7], t0, t1);
    }
  }
  float mx = fmax3f(fmax3f(mxa[0], mxa[1], mxa[2]), fmax3f(mxa[3], mxa[4], mxa[5]), fmaxf(mxa[6], mxa[7]));
  // ---- combine with the other parts of the row.  Two slots alternate: a part rewrites a
  //      slot only after the next rendezvous, which every other part reaches after reading it.
  float* slot = xch + (xc & 1u) * (NSPLIT * 128);
  slot[part * 128 + rloc] = mx;
  mbar_arrive(xbar);
  if (!__all_sync(0xffffffffu, wait_bounded(xbar, xc & 1u, abort_flag, tmo))) return false;
#pragma unroll
  for (int k = 0; k < NSPLIT; ++k) mx = fmaxf(mx, slot[k * 128 + rloc]);
  ++xc;
  if constexpr (kPlain) mx = mx * sc;                  // plain scores are still raw (scale > 0)
  bool rescale = false;
  float alpha = 1.f;
  if (mx > m_run + rescale_tau()) {
    if (m_run != kNegInf) {
      alpha = ex2_approx(m_run - mx);
      rescale = true;
      l_part *= alpha;
    }
    m_run = mx;
  }
#ifdef ATTN_ABLATION
  if (part == 0) {   // one count per (row, key tile) step, as in the single-CTA kernel
    const unsigned r = __ballot_sync(0xffffffffu, rescale), v = __ballot_sync(0xffffffffu, m_run != kNegInf);
    if ((threadIdx.x & 31) == 0) {
      atomicAdd(&g_abl_counts[0], static_cast<unsigned long long>(__popc(r)));
      atomicAdd(&g_abl_counts[1], static_cast<unsigned long long>(__popc(v)));
    }
  }
#endif
  const float msub = (m_run == kNegInf) ? 0.f : m_run;
  const float2 sc2 = make_float2(sc, sc);
  const float2 nm2 = make_float2(-msub, -msub);
  // 2^a; with kSwExpEvery > 0 (ablation build) one pair of key columns in kSwExpEvery goes to
  // the FMA pipes, chosen by the column within the tile as in the single-CTA kernel.
  auto pexp = [&](float a, int c) -> float {
    if (kSwExpEvery > 0 && ((col0 + c) >> 1) % kSwDiv == kSwDiv - 1) {
      const float e = exp2_fma(a);
      return masked ? (a == kNegInf ? 0.f : e) : e;
    }
    return ex2_approx(a);
  };
  float2 ls[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) ls[u] = make_float2(0.f, 0.f);
  uint32_t pk[COLS / 2];
#pragma unroll
  for (int c2 = 0; c2 < COLS / 2; ++c2) {
    const float2 v = make_float2(__uint_as_float(s[2 * c2]), __uint_as_float(s[2 * c2 + 1]));
    const float2 a = kPlain ? ffma2(v, sc2, nm2) : fadd2(v, nm2);
    const float2 pp = make_float2(pexp(a.x, 2 * c2), pexp(a.y, 2 * c2 + 1));
    ls[c2 & 3] = fadd2(ls[c2 & 3], pp);
    pk[c2] = pack_bf16x2(pp.x, pp.y);
  }
  if constexpr (COLS == 64) tmem_st_x32_wait<0>(tS + (COLS / 2) * part, pk);
  else tmem_st_x16_wait<0>(tS + (COLS / 2) * part, pk);
  const float2 l2 = fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3]));
  l_part += l2.x + l2.y;
  // ---- rescale this part of O once P V of the previous key tile is complete
  if (__any_sync(0xffffffffu, rescale)) {
    if (!*prev_done) {
      if (!__all_sync(0xffffffffu, wait_bounded(prev_bar, prev_par, abort_flag, tmo))) return false;
      *prev_done = true;
    }
    tc_fence_after();
#pragma unroll
    for (int ch = 0; ch < COLS / 32; ++ch) {
      uint32_t o[32];
      tmem_ld_x32_wait(tO + col0 + ch * 32, o);
#pragma unroll
      for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
      tmem_st_x32_wait<0>(tO + col0 + ch * 32, o);
    }
  }
  return true;
}

template <int NSPLIT, bool SOFTCAP, bool ALIBI>
__global__ void __launch_bounds__(CfgPair<NSPLIT>::THREADS, 1)
attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = CfgPair<NSPLIT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sptr = smem_raw + (sbase - raw);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sptr + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + C::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();                      // 0: issues the MMAs
  const int G = static_cast<int>(cluster_count_x());           // pairs in the grid
  const int pair = static_cast<int>(cluster_id_x());
  const unsigned long long tmo = p.timeout_ns;

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_QFULL), 1);
    mbar_init(BAR(C::B_QEMPTY), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(BAR(C::B_KVFULL + s), 1);
      mbar_init(BAR(C::B_KVEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(C::B_SFULL + b), 1);
      mbar_init(BAR(C::B_PFULL + b), C::P_ARRIVALS);
    }
    mbar_init(BAR(C::B_ODONE), 1);
    mbar_init(BAR(C::B_DRAIN), 1);
    for (int q = 0; q < 4; ++q) mbar_init(BAR(C::B_XCH + q), 32 * NSPLIT);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc_pair(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == C::LOAD_WARP && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  // Both CTAs' barriers are initialised (and the pair's tensor memory allocated) before any
  // copy, commit or arrival reaches them from the other CTA.
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  if (warp == C::LOAD_WARP) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const bool varlen = p.cu_q != nullptr;
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      uint32_t lidx = 0, qcount = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int w = sched_pos(r, pair, G);
        if (w >= p.num_items) break;
        const Item it = make_item(p, w);
        if (it.n == 0) continue;
        // this CTA's query rows are free once the pair's last S MMA of the previous item is done
        if (qcount > 0 && !wait_bounded(BAR(C::B_QEMPTY), (qcount - 1) & 1, abort_flag, tmo)) break;
        if (rank == 0) mbar_expect_tx(BAR(C::B_QFULL), 2 * C::Q_BYTES);
        const uint32_t qbar = mapa_shared(BAR(C::B_QFULL), 0);
        const int qrow = it.qb * 256 + 128 * static_cast<int>(rank);
        const int qc1 = varlen ? it.h : qrow, qc2 = varlen ? it.q_off + qrow : it.bh;
        for (int pn = 0; pn < 2; ++pn)
          tma_load_3d_pair(sbase + C::OFF_Q + pn * C::QPANEL, &tm_q, qbar, pn * 64, qc1, qc2, pol_q, C::QPANEL);
        ++qcount;
        for (int i = 0; i < it.n && ok; ++i) {
          const int kt = tile_kt(it, i);
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t slot = lidx % C::NS;
            if (kv == 0 && !wait_bounded(BAR(C::B_KVEMPTY + slot), ((lidx / C::NS) & 1) ^ 1, abort_flag, tmo)) {
              ok = false;
              break;
            }
            if (kv == 0 && rank == 0) mbar_expect_tx(BAR(C::B_KVFULL + slot), 2 * C::STAGE);
            const uint32_t kvbar = mapa_shared(BAR(C::B_KVFULL + slot), 0);
            const uint32_t stage = sbase + C::OFF_KV + slot * C::STAGE + kv * C::HALF;
            if (kv == 0) {
              // K: keys 64*rank .. 64*rank+63 of the tile, both 64-column panels
              const int krow = kt * 128 + 64 * static_cast<int>(rank);
              const int kc1 = varlen ? it.kvh : krow, kc2 = varlen ? it.k_off + krow : it.kvbh;
              for (int pn = 0; pn < 2; ++pn)
                tma_load_3d_pair(stage + pn * C::KPANEL, &tm_k, kvbar, pn * 64, kc1, kc2, pol_kv, C::KPANEL);
            } else {
              // V: value columns 64*rank .. 64*rank+63 of all 128 keys of the tile
              const int vc1 = varlen ? it.kvh : kt * 128, vc2 = varlen ? it.k_off + kt * 128 : it.kvbh;
              tma_load_3d_pair(stage, &tm_v, kvbar, 64 * static_cast<int>(rank), vc1, vc2, pol_kv, C::HALF);
            }
          }
          ++lidx;
        }
      }
      // After a time-out some copies may still be in flight, and their completion is counted
      // on the even CTA's barriers, which this thread cannot wait on: give them a fixed,
      // bounded time to land before the CTA can reach its exit.
      if (*abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    if (rank == 0 && lane == 0) {
      const uint32_t tO = tbase + C::T_O;
      auto tS = [&](uint32_t buf) -> uint32_t { return tbase + (buf ? C::T_S1 : C::T_S0); };
      const uint64_t dq = make_sdesc_sw128(sbase + C::OFF_Q, 16, 1024);     // Q: K-major A
      const uint64_t dk = make_sdesc_sw128(sbase + C::OFF_KV, 16, 1024);    // K half: K-major B
      // V half: MN-major B, one 128-byte chunk of columns per CTA (the leading offset is unused)
      const uint64_t dv = make_sdesc_sw128(sbase + C::OFF_KV + C::HALF, C::HALF, 1024);
      auto commit2 = [&](int b) {
        mma_commit_pair(BAR(b));
        mma_commit_pair(mapa_shared(BAR(b), 1));
      };
      auto qk = [&](uint32_t buf, uint32_t slot) {
        const uint64_t b0 = dk + ((slot * C::STAGE) >> 4);
#pragma unroll
        for (int kk = 0; kk < C::D / 16; ++kk) {
          const int col = kk * 16;
          const uint32_t offa = ((col / 64) * C::QPANEL + (col % 64) * 2) >> 4;
          const uint32_t offb = ((col / 64) * C::KPANEL + (col % 64) * 2) >> 4;
          mma_f16_ss_pair(tS(buf), dq + offa, b0 + offb, C::IDESC_QK, kk > 0);
        }
      };
      auto pv = [&](uint32_t buf, uint32_t slot, bool acc) {
        const uint64_t b0 = dv + ((slot * C::STAGE) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ts_pair(tO, tS(buf) + kk * 8, b0 + ((kk * 16 * 128) >> 4), C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
      };
      // The tensor pipe's issue queue is shallow: whatever this thread does between MMAs
      // (waits, commits) leaves the pipe idle.  So each step waits first, then issues P V and
      // the S two tiles ahead back to back, and commits last.
      uint32_t cidx = 0, tcount = 0, qcount = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int w = sched_pos(r, pair, G);
        if (w >= p.num_items) break;
        const Item it = make_item(p, w);
        if (it.n == 0) continue;
        auto full = [&](int j) -> bool {   // key tile j of the item (K and V halves of both CTAs)
          const uint32_t ki = cidx + j;
          return wait_bounded(BAR(C::B_KVFULL + ki % C::NS), (ki / C::NS) & 1, abort_flag, tmo);
        };
        if (!wait_bounded(BAR(C::B_QFULL), qcount & 1, abort_flag, tmo) || !full(0) ||
            (it.n > 1 && !full(1)))
          break;
        tc_fence_after();
        // S(0), S(1) into buffers tcount & 1 and (tcount + 1) & 1
        qk(tcount & 1, cidx % C::NS);
        if (it.n > 1) qk((tcount + 1) & 1, (cidx + 1) % C::NS);
        commit2(C::B_SFULL + (tcount & 1));
        if (it.n > 1) commit2(C::B_SFULL + ((tcount + 1) & 1));
        if (it.n <= 2) commit2(C::B_QEMPTY);   // last read of this item's query rows
        for (int i = 0; i < it.n; ++i) {
          const uint32_t t = tcount + i;
          const bool ahead = i + 2 < it.n;
          // P(i) from both CTAs' softmax warps, and the stage of the S two tiles ahead
          if (!wait_bounded(BAR(C::B_PFULL + (t & 1)), (t >> 1) & 1, abort_flag, tmo) || (ahead && !full(i + 2))) {
            ok = false;
            break;
          }
          tc_fence_after();
          pv(t & 1, (cidx + i) % C::NS, i > 0);
          // S(i+2) overwrites P(i) in its buffer: the pair's MMAs execute in issue order
          if (ahead) qk(t & 1, (cidx + i + 2) % C::NS);
          if (ahead) commit2(C::B_SFULL + (t & 1));
          if (ahead && i + 2 == it.n - 1) commit2(C::B_QEMPTY);
          commit2(C::B_KVEMPTY + (cidx + i) % C::NS);   // stage of tile i: K read by S(i), V by P V(i)
          // P V done for the last two tiles (the softmax's rescale before its last P, and the
          // epilogue); earlier ones are implied by the completion of the S issued after them
          if (i + 2 >= it.n) commit2(C::B_ODONE);
        }
        if (!ok) break;
        cidx += it.n;
        tcount += it.n;
        ++qcount;
      }
      // every pair MMA issued here is complete before the pair's tensor memory is freed
      mma_commit_pair(BAR(C::B_DRAIN));
      drain_bounded(BAR(C::B_DRAIN), 0, tmo);
    }
  } else if (warp < 4 * NSPLIT) {
    // ------------------------------------------------------------------ softmax (both CTAs)
    const int quarter = warp & 3, part = warp >> 2;
    const int rloc = quarter * 32 + lane;                   // query row within this CTA's 128 (TMEM lane)
    constexpr int COLS = C::COLS;
    const int col0 = COLS * part;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tO = tbase + C::T_O + lane_off;
    const int g = static_cast<int>(rank);                   // this CTA's query tile of the item
    float* xch = reinterpret_cast<float*>(sptr + C::OFF_XCH);
    const uint32_t xbar = BAR(C::B_XCH + quarter);
    const uint32_t obar = BAR(C::B_ODONE);
    const uint32_t pbar0 = mapa_shared(BAR(C::B_PFULL), 0), pbar1 = mapa_shared(BAR(C::B_PFULL + 1), 0);
    const bool has_doc = (p.mask_kind & 4) != 0;
    uint32_t tcount = 0, xc = 0, od = 0;   // tiles, rendezvous and o_done phases seen
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int w = sched_pos(r, pair, G);
      if (w >= p.num_items) break;
      const Item it = make_item(p, w);
      const int row = it.qb * 256 + 128 * g + rloc;
      const int ip = row + (it.sk - it.sq);
      int jlo_row = lo_key(p, ip);
      int jhi_row = hi_key(p, it.sk, ip);
      const int doc_row = (has_doc && row < p.Sq) ? __ldg(p.doc + static_cast<size_t>(it.b) * p.Sk + row) : 0;
      bool doc_elem = has_doc;
      if (has_doc && p.doc_sorted != nullptr && __ldg(p.doc_sorted + it.b) != 0) {
        if (row < p.Sq) {
          const int* drow = p.doc + static_cast<size_t>(it.b) * p.Sk;
          int lo = 0, hi = p.Sk;
          while (lo < hi) { const int mid = (lo + hi) >> 1; if (__ldg(drow + mid) < doc_row) lo = mid + 1; else hi = mid; }
          const int ds = lo;
          hi = p.Sk;
          while (lo < hi) { const int mid = (lo + hi) >> 1; if (__ldg(drow + mid) <= doc_row) lo = mid + 1; else hi = mid; }
          jlo_row = max(jlo_row, ds);
          jhi_row = min(jhi_row, lo - 1);
        }
        doc_elem = false;
      }
      float slope_l2 = 0.f;
      if constexpr (ALIBI) slope_l2 = __ldg(p.alibi + it.h) * kLog2e;
      float m_run = kNegInf, l_part = 0.f;
      for (int i = 0; i < it.n; ++i) {
        const uint32_t t = tcount + i;
        const uint32_t tS = tbase + ((t & 1) ? C::T_S1 : C::T_S0) + lane_off;
        const int kt = tile_kt(it, i);
        const int cls = tile_class(p, it, i, g, kt);
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_SFULL + (t & 1)), (t >> 1) & 1, abort_flag, tmo))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // Completion of P V(i-1), needed before O is rescaled: implied by S(i+1), which the MMA
        // issues after it; for the item's last tile, o_done (committed after P V(n-2)).  At
        // i = 0 the running maximum is still -inf, so no rescale can occur.
        const bool last = (i + 1 == it.n);
        bool prev_done = (i == 0);
        const uint32_t prev_bar = last ? obar : BAR(C::B_SFULL + ((t + 1) & 1));
        const uint32_t prev_par = last ? (od & 1u) : (((t + 1) >> 1) & 1u);
        if (cls == 0) {
          uint32_t z[COLS / 2];
#pragma unroll
          for (int c = 0; c < COLS / 2; ++c) z[c] = 0u;
          if constexpr (COLS == 64) tmem_st_x32_wait<0>(tS + (COLS / 2) * part, z);   // P = 0 for this part
          else tmem_st_x16_wait<0>(tS + (COLS / 2) * part, z);
        } else if (!softmax_part<NSPLIT, SOFTCAP, ALIBI>(p, it, kt, cls, part, rloc, tS, tO, ip, jlo_row, jhi_row,
                                                         doc_elem, doc_row, slope_l2, xch, xbar, xc, prev_bar,
                                                         prev_par, &prev_done, t, abort_flag, tmo, m_run, l_part)) {
          ok = false;
          break;
        }
        // the o_done phase of P V(n-2) is consumed before P(n-1) is signalled, so that o_done
        // is never two phases ahead of the phase waited for
        if (last && i > 0) {
          if (!prev_done && !__all_sync(0xffffffffu, wait_bounded(obar, od & 1u, abort_flag, tmo))) {
            ok = false;
            break;
          }
          ++od;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && !(p.fault_skip && rank == 1 && warp == 0 && t == 0)) mbar_arrive_remote((t & 1) ? pbar1 : pbar0);
      }
      if (!__all_sync(0xffffffffu, ok && !*abort_flag)) {
        ok = false;
        break;
      }
      // ---- epilogue: O / l -> bf16 (this part's columns), LSE (part 0); every part adds the
      //      partial sums in the same order, so all parts of a row scale by the same l
      if (it.n > 0) {   // P V(n-1) complete
        if (!__all_sync(0xffffffffu, wait_bounded(obar, od & 1u, abort_flag, tmo))) {
          ok = false;
          break;
        }
        ++od;
        tc_fence_after();
      }
      float* slot = xch + (xc & 1u) * (NSPLIT * 128);
      slot[part * 128 + rloc] = l_part;
      mbar_arrive(xbar);
      if (!__all_sync(0xffffffffu, wait_bounded(xbar, xc & 1u, abort_flag, tmo))) {
        ok = false;
        break;
      }
      float l_run = 0.f;
#pragma unroll
      for (int k = 0; k < NSPLIT; ++k) l_run += slot[k * 128 + rloc];
      ++xc;
      const float inv_l = (l_run > 0.f) ? (1.f / l_run) : 0.f;
      const bool varlen = p.cu_q != nullptr;
      const size_t orow_idx = varlen ? static_cast<size_t>(it.q_off + row) * p.H + it.h
                                     : static_cast<size_t>(it.bh) * p.Sq + row;
      const size_t lse_idx = varlen ? static_cast<size_t>(it.h) * p.Tq + it.q_off + row
                                    : static_cast<size_t>(it.bh) * p.Sq + row;
      __nv_bfloat16* orow = p.o + orow_idx * C::D + col0;
#pragma unroll
      for (int ch = 0; ch < COLS / 32; ++ch) {
        uint32_t o[32];
        if (it.n > 0) {
          tmem_ld_x32_wait(tO + col0 + ch * 32, o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        uint32_t wv[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          wv[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
        if (row < it.sq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) __stcs(dst + v, make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]));
        }
      }
      if (part == 0 && row < it.sq) {
        const float lse = (l_run > 0.f) ? (m_run + lg2_approx(l_run)) * kLn2 : kNegInf;
        p.lse[lse_idx] = lse;
      }
      tcount += it.n;
    }
  }

  // ------------------------------------------------------------------ teardown (both CTAs)
  tc_fence_before();
  cluster_sync_all();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, C::TMEM_COLS);
  }
}

}  // namespace attn
