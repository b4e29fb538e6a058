// attn_fwd_kernel.cuh — fused attention forward for sm_100a (B200).
//
// What it computes: O = softmax(score_mod(scale * Q K^T), masked) V and the per-row
// log-sum-exp, tile by tile with an online softmax that keeps only a running maximum and
// a running sum per query row, so the score matrix never reaches HBM (page "FlashAttention
// 4: Γρηγορότερη και Αποδοτική σε Μνήμη Προσοχή για LLMs", sections "Εισαγωγή" and
// "Γιατί οι πυρήνες προσοχής ..."; the FlexAttention variants from the page "PyTorch's
// FlexAttention mit FlashAttention-4 ist ein Game-Changer", intro).
//
// Work item: one (b, h) and one block of 256 query rows, made of two 128-row query tiles
// (the 256x128 Blackwell tile shape named on the FlexAttention page, section "Aktuelle
// Einschränkungen").  One CTA per work item, 10 warps:
//   warps 0-3  softmax group 0: one thread per row of query tile 0
//   warps 4-7  softmax group 1: one thread per row of query tile 1
//   warp  8    TMA producer: Q tiles once, then a ring of K and V tiles
//   warp  9    MMA issuer (one thread): S_g = Q_g K^T and O_g += P_g V with tcgen05, both
//              accumulating in tensor memory; also allocates / frees TMEM.
// Tensor memory (512 columns): S0 | S1 | O0 | O1.  P_g (bf16 or e4m3) is written over the
// first columns of S_g once the thread has read its whole S row.
//
// The two groups ping-pong on the tensor core (S0, PV1, S1, PV0, ...) so that one group's
// exponentials overlap the other group's MMAs — the producer/consumer split and overlap of
// block GEMM and softmax described on the page "FlashAttention-3: ...", section "Analyse",
// re-done for tcgen05 (one issuing thread, accumulators in TMEM, mbarrier hand-offs).
//
// Online softmax with a rescale threshold (page "FlashAttention 4 ...", section "Έξυπνος
// επανακανονισμός Softmax στο Διαδίκτυο"): the running maximum m used for the
// exponentials is only raised when a new row maximum exceeds it by more than TAU (log2
// units); otherwise exponentials are taken against the stale m, which is exact in real
// arithmetic because O and the row sum l share that m.  TAU = 8 keeps P <= 256, which
// bf16 and e4m3 represent.
//
// Every wait is bounded (global timer); on time-out the kernel records ATTN_ERR_TIMEOUT in
// the device status word, all roles unwind, in-flight TMA copies and MMAs are drained
// (again with a bound), TMEM is freed, and the CTA returns.  Nothing traps.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace attn {

constexpr int kThreads = 320;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kTau = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNegInf = -__builtin_huge_valf();

// Device status word (one per device that loads the library).
__device__ int g_attn_status;

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  int B, H, Sq, Sk;
  int nqb, nkt;            // 256-row query blocks, 128-column key tiles
  int mask_kind, window;   // window already clamped to <= Sq + Sk
  float scale_log2;        // scale * log2(e)
  float sc_in, sc_out;     // soft-capping: x = s * sc_in, t = tanh(x) * sc_out (log2 units)
  const float* alibi;      // [H] slopes or nullptr
  const int* doc;          // [B, Sk] or nullptr
  const int* map_counts;   // [B, nqb] or nullptr (analytic ranges)
  const uint32_t* map_entries;  // [B, nqb, nkt]
  // FP8 block scales [B, H, nsb] (nullptr for bf16)
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  int nsb_q, nsb_k;
  int fault_skip;          // test hook: group 1 skips its first P-ready signal
  unsigned long long timeout_ns;
};

template <int D, bool FP8>
struct Cfg {
  static constexpr int EB = FP8 ? 1 : 2;                 // element bytes
  static constexpr int PANEL_COLS = 128 / EB;            // columns per 128-byte swizzle panel
  static constexpr int NPANEL = D / PANEL_COLS;
  static constexpr int PANEL_BYTES = 128 * 128;          // 128 rows x 128 bytes
  static constexpr int TILE_BYTES = 128 * D * EB;        // one 128-row tile of Q, K or V
  static constexpr int KSTEP = 32 / EB;                  // MMA K per instruction (32 bytes)
  static constexpr int QK_STEPS = D / KSTEP;
  static constexpr int PV_STEPS = 128 / KSTEP;
  static constexpr int P_COLS = 128 * EB / 4;            // TMEM columns holding one P row
  static constexpr int NS = (TILE_BYTES >= 32768) ? 4 : 8;   // K/V ring depth
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NS * TILE_BYTES;
  // barriers: q_full[2], kv_full[NS], kv_empty[NS], s_full[2], p_full[2], o_done[2], drain
  static constexpr int NBAR = 2 + 2 * NS + 2 + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;    // tmem base (4 B), abort flag (4 B)
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S0 = 0, T_S1 = 128, T_O0 = 256, T_O1 = 256 + D;
  static constexpr uint32_t IDESC_QK = make_idesc(FP8 ? 0u : 1u, 128, 128, false);
  static constexpr uint32_t IDESC_PV = make_idesc(FP8 ? 0u : 1u, 128, D, true);
};

// ---------------------------------------------------------------------------------------
// bounded waiting
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void record_timeout() {
  atomicCAS(&g_attn_status, 0, -4 /* ATTN_ERR_TIMEOUT */);
}

// Waits for phase `parity` of the barrier.  Returns false (and raises the CTA abort flag)
// when the time limit runs out or another role has already aborted.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             unsigned long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > timeout_ns) {
        *abort_flag = 1;
        record_timeout();
        return false;
      }
    }
  }
}

// Waits without giving up on another role's abort (used to drain this role's own copies
// and MMAs before TMEM is freed); still bounded by the time limit.
__device__ __forceinline__ bool drain_bounded(uint32_t bar, uint32_t parity,
                                              unsigned long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0 && global_timer_ns() - t0 > timeout_ns) {
      record_timeout();
      return false;
    }
  }
}

// ---------------------------------------------------------------------------------------
// tile schedule
// ---------------------------------------------------------------------------------------
struct Item {
  int b, h, bh, qb;
  int n;          // number of key tiles visited
  int kt_lo;      // analytic: first key tile
  const uint32_t* entries;  // map: entry list (nullptr for analytic)
};

__device__ __forceinline__ int hi_key(const FwdParams& p, int ip) {  // last visible key of row i'
  int h = (p.mask_kind & 1) ? ip : ((p.mask_kind & 2) ? ip + p.window - 1 : p.Sk - 1);
  return min(h, p.Sk - 1);
}
__device__ __forceinline__ int lo_key(const FwdParams& p, int ip) {  // first visible key (unclipped)
  return (p.mask_kind & 2) ? ip - p.window + 1 : 0;
}

__device__ __forceinline__ Item make_item(const FwdParams& p, int item) {
  Item it;
  it.bh = item / p.nqb;
  it.qb = p.nqb - 1 - item % p.nqb;   // longest first within a head (causal)
  it.b = it.bh / p.H;
  it.h = it.bh % p.H;
  it.entries = nullptr;
  it.kt_lo = 0;
  if (p.map_counts != nullptr) {
    it.n = p.map_counts[it.b * p.nqb + it.qb];
    it.entries = p.map_entries + (static_cast<size_t>(it.b) * p.nqb + it.qb) * p.nkt;
    return it;
  }
  const int d = p.Sk - p.Sq;
  int A = it.qb * 256 + d;
  const int Bm = min(it.qb * 256 + 255, p.Sq - 1) + d;
  if (p.mask_kind & 1) A = max(A, 0);
  const int klo = max(0, lo_key(p, A));
  const int khi = hi_key(p, Bm);
  if (((p.mask_kind & 1) && Bm < 0) || khi < klo) {
    it.n = 0;
    return it;
  }
  it.kt_lo = klo / 128;
  it.n = khi / 128 + 1 - it.kt_lo;
  return it;
}

__device__ __forceinline__ int tile_kt(const Item& it, int i) {
  return it.entries ? static_cast<int>(__ldg(it.entries + i) & 0xFFFFFFu) : it.kt_lo + i;
}

// Class of (query tile g, key tile kt): 0 EMPTY, 1 PARTIAL, 2 FULL.
__device__ __forceinline__ int tile_class(const FwdParams& p, const Item& it, int i, int g, int kt) {
  if (it.entries) return static_cast<int>((__ldg(it.entries + i) >> (24 + 2 * g)) & 3u);
  const int r0 = it.qb * 256 + 128 * g;
  if (r0 >= p.Sq) return 0;
  const int r1 = min(r0 + 127, p.Sq - 1);
  const int d = p.Sk - p.Sq;
  const int a = r0 + d, bb = r1 + d;
  const int c0 = kt * 128, c1 = c0 + 127, c1v = min(c1, p.Sk - 1);
  const bool causal = p.mask_kind & 1, win = p.mask_kind & 2;
  const int i1 = causal ? c0 : (win ? c0 - p.window + 1 : INT_MIN);
  const int i2 = win ? c1v + p.window - 1 : INT_MAX;
  if (max(a, i1) > min(bb, i2)) return 0;
  const bool full = (c1 <= p.Sk - 1) && (!win || bb - p.window + 1 <= c0) &&
                    (causal ? (a >= c1) : (!win || a + p.window - 1 >= c1));
  return full ? 2 : 1;
}

// ---------------------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------------------
template <int D, bool FP8, bool SOFTCAP, bool ALIBI>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = Cfg<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sptr = smem_raw + (sbase - raw);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
  const int B_QFULL = 0, B_KVFULL = 2, B_KVEMPTY = 2 + C::NS, B_SFULL = 2 + 2 * C::NS,
            B_PFULL = B_SFULL + 2, B_ODONE = B_PFULL + 2, B_DRAIN = B_ODONE + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sptr + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Item it = make_item(p, blockIdx.x);
  const unsigned long long tmo = p.timeout_ns;

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_QFULL + 0), 1);
    mbar_init(BAR(B_QFULL + 1), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(BAR(B_KVFULL + s), 1);
      mbar_init(BAR(B_KVEMPTY + s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(BAR(B_SFULL + g), 1);
      mbar_init(BAR(B_PFULL + g), 128);
      mbar_init(BAR(B_ODONE + g), 1);
    }
    mbar_init(BAR(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  if (warp == kLoadWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      for (int g = 0; g < 2; ++g) {
        mbar_expect_tx(BAR(B_QFULL + g), C::TILE_BYTES);
        for (int pn = 0; pn < C::NPANEL; ++pn)
          tma_load_3d(sbase + C::OFF_Q + g * C::TILE_BYTES + pn * C::PANEL_BYTES, &tm_q,
                      BAR(B_QFULL + g), pn * C::PANEL_COLS, it.qb * 256 + 128 * g, it.bh, pol_q);
      }
      int issued = 0;  // loads issued into the ring
      for (int i = 0; i < it.n; ++i) {
        const int kt = tile_kt(it, i);
        bool ok = true;
        for (int kv = 0; kv < 2 && ok; ++kv) {
          const int idx = 2 * i + kv;
          const int slot = idx % C::NS;
          const uint32_t par = ((idx / C::NS) & 1) ^ 1;
          if (!wait_bounded(BAR(B_KVEMPTY + slot), par, abort_flag, tmo)) {
            ok = false;
            break;
          }
          mbar_expect_tx(BAR(B_KVFULL + slot), C::TILE_BYTES);
          const CUtensorMap* tm = kv ? &tm_v : &tm_k;
          for (int pn = 0; pn < C::NPANEL; ++pn)
            tma_load_3d(sbase + C::OFF_KV + slot * C::TILE_BYTES + pn * C::PANEL_BYTES, tm,
                        BAR(B_KVFULL + slot), pn * C::PANEL_COLS, kt * 128, it.bh, pol_kv);
          ++issued;
        }
        if (!ok) break;
      }
      // Drain: every copy issued by this thread has landed before the CTA may exit.
      drain_bounded(BAR(B_QFULL + 0), 0, tmo);
      drain_bounded(BAR(B_QFULL + 1), 0, tmo);
      for (int idx = max(0, issued - C::NS); idx < issued; ++idx)
        drain_bounded(BAR(B_KVFULL + idx % C::NS), (idx / C::NS) & 1, tmo);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS[2] = {tbase + C::T_S0, tbase + C::T_S1};
      const uint32_t tO[2] = {tbase + C::T_O0, tbase + C::T_O1};
      const uint32_t sQ[2] = {sbase + C::OFF_Q, sbase + C::OFF_Q + C::TILE_BYTES};
      auto qk = [&](int g, int kslot) {
        const uint32_t kbase = sbase + C::OFF_KV + kslot * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::QK_STEPS; ++kk) {
          const int col = kk * C::KSTEP;
          const uint32_t off = (col / C::PANEL_COLS) * C::PANEL_BYTES + (col % C::PANEL_COLS) * C::EB;
          const uint64_t ad = make_sdesc_sw128(sQ[g] + off, 16, 1024);
          const uint64_t bd = make_sdesc_sw128(kbase + off, 16, 1024);
          if constexpr (FP8) mma_f8_ss(tS[g], ad, bd, C::IDESC_QK, kk > 0);
          else mma_f16_ss(tS[g], ad, bd, C::IDESC_QK, kk > 0);
        }
      };
      auto pv = [&](int g, int vslot, bool acc) {
        const uint32_t vbase = sbase + C::OFF_KV + vslot * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::PV_STEPS; ++kk) {
          const uint64_t bd = make_sdesc_sw128(vbase + kk * C::KSTEP * 128, C::PANEL_BYTES, 1024);
          const uint32_t ta = tS[g] + kk * (C::KSTEP * C::EB / 4);
          if constexpr (FP8) mma_f8_ts(tO[g], ta, bd, C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
          else mma_f16_ts(tO[g], ta, bd, C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = wait_bounded(BAR(B_QFULL + 0), 0, abort_flag, tmo) &&
                wait_bounded(BAR(B_QFULL + 1), 0, abort_flag, tmo);
      int prev_vslot = 0;
      for (int i = 0; i < it.n && ok; ++i) {
        const int kidx = 2 * i, vidx = 2 * i + 1;
        const int kslot = kidx % C::NS, vslot = vidx % C::NS;
        // S0(i) = Q0 K_i^T   (S0 holds P0(i-1) until PV0(i-1) has completed)
        if (!wait_bounded(BAR(B_KVFULL + kslot), (kidx / C::NS) & 1, abort_flag, tmo)) break;
        if (i > 0 && !wait_bounded(BAR(B_ODONE + 0), (i - 1) & 1, abort_flag, tmo)) break;
        tc_fence_after();
        qk(0, kslot);
        mma_commit(BAR(B_SFULL + 0));
        // O1 += P1(i-1) V_{i-1}
        if (i > 0) {
          if (!wait_bounded(BAR(B_PFULL + 1), (i - 1) & 1, abort_flag, tmo)) { ok = false; break; }
          tc_fence_after();
          pv(1, prev_vslot, i - 1 > 0);
          mma_commit(BAR(B_ODONE + 1));
          mma_commit(BAR(B_KVEMPTY + prev_vslot));
          if (!wait_bounded(BAR(B_ODONE + 1), (i - 1) & 1, abort_flag, tmo)) { ok = false; break; }
          tc_fence_after();
        }
        // S1(i) = Q1 K_i^T
        qk(1, kslot);
        mma_commit(BAR(B_SFULL + 1));
        mma_commit(BAR(B_KVEMPTY + kslot));
        // O0 += P0(i) V_i
        if (!wait_bounded(BAR(B_KVFULL + vslot), (vidx / C::NS) & 1, abort_flag, tmo)) break;
        if (!wait_bounded(BAR(B_PFULL + 0), i & 1, abort_flag, tmo)) break;
        tc_fence_after();
        pv(0, vslot, i > 0);
        mma_commit(BAR(B_ODONE + 0));
        prev_vslot = vslot;
      }
      if (ok && it.n > 0 && !*abort_flag) {
        // O1 += P1(n-1) V_{n-1}
        if (wait_bounded(BAR(B_PFULL + 1), (it.n - 1) & 1, abort_flag, tmo)) {
          tc_fence_after();
          pv(1, prev_vslot, it.n - 1 > 0);
          mma_commit(BAR(B_ODONE + 1));
          mma_commit(BAR(B_KVEMPTY + prev_vslot));
        }
      }
      // Drain: all MMAs issued by this thread are complete before TMEM is freed.
      mma_commit(BAR(B_DRAIN));
      drain_bounded(BAR(B_DRAIN), 0, tmo);
    }
  } else {
    // ------------------------------------------------------------------ softmax groups
    const int g = warp >> 2;                       // query tile of this group
    const int rloc = (warp & 3) * 32 + lane;       // row within the query tile (= TMEM lane)
    const int row = it.qb * 256 + 128 * g + rloc;  // query row
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + (g ? C::T_S1 : C::T_S0) + lane_off;
    const uint32_t tO = tbase + (g ? C::T_O1 : C::T_O0) + lane_off;
    const int ip = row + (p.Sk - p.Sq);            // bottom-right aligned position
    const int jlo_row = lo_key(p, ip);
    const int jhi_row = hi_key(p, ip);
    const bool has_doc = (p.mask_kind & 4) != 0;
    const int doc_row = (has_doc && row < p.Sq) ? __ldg(p.doc + static_cast<size_t>(it.b) * p.Sk + row) : 0;
    float slope_l2 = 0.f;
    if constexpr (ALIBI) slope_l2 = __ldg(p.alibi + it.h) * kLog2e;
    float sq_scale = 1.f, v_norm = 1.f;
    if constexpr (FP8) {
      const size_t qbase = static_cast<size_t>(it.bh) * p.nsb_q;
      sq_scale = __ldg(p.q_scale + qbase + min(2 * it.qb + g, p.nsb_q - 1));
      const size_t vbase = static_cast<size_t>(it.bh) * p.nsb_k;
      float vm = 0.f;
      for (int sb = 0; sb < p.nsb_k; ++sb) vm = fmaxf(vm, __ldg(p.v_scale + vbase + sb));
      v_norm = vm > 0.f ? vm : 1.f;
    }

    float m_run = kNegInf;   // running maximum used for the exponentials (log2 units)
    float l_run = 0.f;       // running row sum against m_run
    bool ok = true;
    for (int i = 0; i < it.n; ++i) {
      const int kt = tile_kt(it, i);
      const int cls = tile_class(p, it, i, g, kt);
      if (!wait_bounded(BAR(B_SFULL + g), i & 1, abort_flag, tmo)) { ok = false; break; }
      tc_fence_after();
      if (cls == 0) {
        // Fully masked for this query tile: P = 0, m and l unchanged.
        uint32_t z[C::P_COLS];
#pragma unroll
        for (int c = 0; c < C::P_COLS; ++c) z[c] = 0u;
        if constexpr (C::P_COLS == 64) tmem_st_x64_wait(tS, z);
        else tmem_st_x32_wait(tS, z);
      } else {
        uint32_t s[128];
        tmem_ld_x128_wait(tS, s);
        float sc = p.scale_log2;     // raw score -> log2 units
        float sc_in = p.sc_in;       // raw score -> tanh argument
        float pv_factor = 1.f;
        if constexpr (FP8) {
          const size_t kb = static_cast<size_t>(it.bh) * p.nsb_k + kt;
          const float sqk = sq_scale * __ldg(p.k_scale + kb);
          sc *= sqk;
          sc_in *= sqk;
          pv_factor = __ldg(p.v_scale + kb) / v_norm;
        }
        const int c0 = kt * 128;
        // ---- score_mod (log2 units) and mask; row maximum
        float mx = kNegInf;
        constexpr bool kPlain = !SOFTCAP && !ALIBI;
        if (cls == 1) {
          const int clo = jlo_row - c0, chi = jhi_row - c0;
          const int* dk = p.doc + static_cast<size_t>(it.b) * p.Sk + c0;
          const int nvalid = p.Sk - c0;
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            float t = __uint_as_float(s[c]);
            if constexpr (!kPlain) {
              if constexpr (SOFTCAP) {
                const float x = t * sc_in;
                const float e = ex2_approx(fabsf(x) * (2.f * kLog2e));
                t = copysignf(1.f - 2.f * rcp_approx(e + 1.f), x) * p.sc_out;
              } else {
                t *= sc;
              }
              if constexpr (ALIBI) t = fmaf(slope_l2, static_cast<float>(c), t + slope_l2 * static_cast<float>(c0 - ip));
            }
            bool vis = (c >= clo) && (c <= chi);
            if (has_doc) vis = vis && (c < nvalid) && (__ldg(dk + min(c, nvalid - 1)) == doc_row);
            t = vis ? t : kNegInf;
            s[c] = __float_as_uint(t);
            mx = fmaxf(mx, t);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            float t = __uint_as_float(s[c]);
            if constexpr (!kPlain) {
              if constexpr (SOFTCAP) {
                const float x = t * sc_in;
                const float e = ex2_approx(fabsf(x) * (2.f * kLog2e));
                t = copysignf(1.f - 2.f * rcp_approx(e + 1.f), x) * p.sc_out;
              } else {
                t *= sc;
              }
              if constexpr (ALIBI) t = fmaf(slope_l2, static_cast<float>(c), t + slope_l2 * static_cast<float>(c0 - ip));
              s[c] = __float_as_uint(t);
            }
            mx = fmaxf(mx, t);
          }
        }
        // In the plain case the scores are still raw: scale the maximum (scale > 0).
        if constexpr (kPlain) mx = mx * sc;
        // ---- online softmax with the rescale threshold
        bool rescale = false;
        float alpha = 1.f;
        if (mx > m_run + kTau) {
          if (m_run != kNegInf) {
            alpha = ex2_approx(m_run - mx);
            rescale = true;
            l_run *= alpha;
          }
          m_run = mx;
        }
        const float msub = (m_run == kNegInf) ? 0.f : m_run;
        float l0 = 0.f, l1 = 0.f;
        uint32_t pk[C::P_COLS];
        if constexpr (!FP8) {
#pragma unroll
          for (int c2 = 0; c2 < 64; ++c2) {
            float a0, a1;
            if constexpr (kPlain) {
              a0 = fmaf(__uint_as_float(s[2 * c2]), sc, -msub);
              a1 = fmaf(__uint_as_float(s[2 * c2 + 1]), sc, -msub);
            } else {
              a0 = __uint_as_float(s[2 * c2]) - msub;
              a1 = __uint_as_float(s[2 * c2 + 1]) - msub;
            }
            const float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
            l0 += p0;
            l1 += p1;
            pk[c2] = pack_bf16x2(p0, p1);
          }
          tmem_st_x64_wait(tS, pk);
        } else {
#pragma unroll
          for (int c4 = 0; c4 < 32; ++c4) {
            float pp[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              float a;
              if constexpr (kPlain) a = fmaf(__uint_as_float(s[4 * c4 + u]), sc, -msub);
              else a = __uint_as_float(s[4 * c4 + u]) - msub;
              pp[u] = ex2_approx(a);
            }
            l0 += pp[0] + pp[2];
            l1 += pp[1] + pp[3];
            pk[c4] = pack_e4m3x2(pp[0] * pv_factor, pp[1] * pv_factor) |
                     (pack_e4m3x2(pp[2] * pv_factor, pp[3] * pv_factor) << 16);
          }
          tmem_st_x32_wait(tS, pk);
        }
        l_run += l0 + l1;
        // ---- rescale O when the maximum moved by more than TAU (PV_g(i-1) is complete:
        //      its commit preceded the one that signalled S_g(i)).
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t o[32];
            tmem_ld_x32_wait(tO + ch * 32, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st_x32_wait(tO + ch * 32, o);
          }
        }
      }
      tc_fence_before();
      if (!(p.fault_skip && g == 1 && i == 0)) mbar_arrive(BAR(B_PFULL + g));
    }
    // ---- epilogue: O / l -> bf16, LSE
    if (ok && !*abort_flag) {
      bool have = true;
      if (it.n > 0) have = wait_bounded(BAR(B_ODONE + g), (it.n - 1) & 1, abort_flag, tmo);
      if (have) {
        tc_fence_after();
        const float inv_l = (l_run > 0.f) ? (v_norm / l_run) : 0.f;
        __nv_bfloat16* orow = p.o + (static_cast<size_t>(it.bh) * p.Sq + row) * D;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          if (it.n > 0) {
            tmem_ld_x32_wait(tO + ch * 32, o);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = 0u;
          }
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            w[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
          if (row < p.Sq) {
            uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          }
        }
        if (row < p.Sq) {
          const float lse = (l_run > 0.f) ? (m_run + lg2_approx(l_run)) * kLn2 : kNegInf;
          p.lse[static_cast<size_t>(it.bh) * p.Sq + row] = lse;
        }
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace attn
