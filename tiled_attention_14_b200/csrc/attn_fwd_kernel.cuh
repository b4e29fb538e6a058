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
// Einschränkungen").  Persistent: one CTA per SM walks a static share of the work items.
// 12 warps:
//   warps 0-3  softmax group 0: one thread per row of query tile 0
//   warps 4-7  softmax group 1: one thread per row of query tile 1
//   warp  8    TMA producer: the item's Q tiles, then a ring of K and V tiles (no L2
//              prefetches: measured, they delay the loads behind them in the TMA unit)
//   warp  9    MMA issuer (one thread): S_g = Q_g K^T and O_g += P_g V with tcgen05, both
//              accumulating in tensor memory; also allocates / frees TMEM
//   warps 10-11 idle (their warpgroup's registers go to the softmax warpgroups).
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

constexpr int kThreads = 384;          // three warpgroups
// Register split (setmaxnreg): the kernel is launched with kLaunchRegs per thread
// (384 x 168 = 64512 of the SM's 65536); the producer/MMA warpgroup gives registers back
// and the two softmax warpgroups take them: 256 x 200 + 128 x 104 = 64512.  The build
// checks that ptxas assigned exactly kLaunchRegs, otherwise an increase could never be met.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 200;
constexpr int kControlRegs = 104;
static_assert(256 * kSoftmaxRegs + 128 * kControlRegs == kThreads * kLaunchRegs, "register split");
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kTau = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNegInf = -__builtin_huge_valf();

// Software exp2 (FMA pipes) takes one element pair in kSwExpEvery (0: all on MUFU).  Measured on
// B200: with the packed-f32x2 softmax the exponentials are not MUFU-bound, so the product build
// has it off; the ablation build (ATTN_ABLATION) compiles it in with ATTN_SW_EXP_EVERY.
#ifndef ATTN_SW_EXP_EVERY
#define ATTN_SW_EXP_EVERY 0
#endif
constexpr int kSwExpEvery = ATTN_SW_EXP_EVERY;
constexpr int kSwDiv = kSwExpEvery > 0 ? kSwExpEvery : 1;
// Coefficients of 2^f on [-1/2, 1/2] (near-minimax in relative error, fitted by
// tiled_attention_14_b200/fit_exp2_poly.py; max relative error 7.5e-5 in float32).
constexpr float kE0 = 0.9999280571937561f;
constexpr float kE1 = 0.6932609677314758f;
constexpr float kE2 = 0.2426111400127411f;
constexpr float kE3 = 0.0551716685295105f;


#ifdef ATTN_ABLATION
// Ablation build only: the rescale threshold comes from device memory, and every (row, key
// tile) step of the softmax is counted — [0] steps that rescaled, [1] steps of rows that had
// seen a visible key.
__device__ float g_abl_tau = 8.0f;
__device__ unsigned long long g_abl_counts[2];
#endif
__device__ __forceinline__ float rescale_tau() {
#ifdef ATTN_ABLATION
  return *reinterpret_cast<volatile float*>(&g_abl_tau);
#else
  return kTau;
#endif
}

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  int B, H, Sq, Sk;        // packed sequences: Sq, Sk are the longest query / key lengths
  int Hkv, group;          // key/value heads; query head h reads key/value head h / group
  int nqb, nkt;            // 256-row query blocks, 128-column key tiles (per sequence)
  // Packed variable-length sequences (token-major [T, H, D] tensors, LSE [H, Tq]):
  // sequence s owns tokens cu_q[s] .. cu_q[s+1]-1 (queries) and cu_k[s] .. cu_k[s+1]-1 (keys).
  const int* cu_q;         // [nseq + 1] or nullptr (batched [B, H, S, D] tensors)
  const int* cu_k;
  int Tq, Tk;              // total query / key tokens (LSE layout [H, Tq])
  int mask_kind, window;   // window already clamped to <= Sq + Sk
  float scale_log2;        // scale * log2(e)
  float sc_in, sc_out;     // soft-capping: x = s * sc_in, t = tanh(x) * sc_out (log2 units)
  const float* alibi;      // [H] slopes or nullptr
  const int* doc;          // [B, Sk] or nullptr
  const int* doc_sorted;   // [B]: 1 if doc[b, :] is non-decreasing (from the tile-map build), or nullptr
  const int* map_counts;   // [B, nqb] or nullptr (analytic ranges)
  const uint32_t* map_entries;  // [B, nqb, nkt]
  // FP8 block scales [B, H, nsb] (nullptr for bf16)
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  int nsb_q, nsb_k;
  int num_items;           // B * H * nqb work items
  int lpt_qb_major;        // 1: order work by query block first (causal: longest first)
  int lpt_heads;           // ... within groups of this many (b, h) heads (0: one group)
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
  // barriers: q_full[2], kv_full[NS], kv_empty[NS], s_full[2], p_full[2], o_done[2], drain, q_empty[2]
  static constexpr int NBAR = 2 + 2 * NS + 2 + 2 + 2 + 1 + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;    // tmem base (4 B), abort flag (4 B)
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S0 = 0, T_S1 = 128, T_O0 = 256, T_O1 = 256 + D;
  static constexpr uint32_t IDESC_QK = make_idesc(FP8 ? 0u : 1u, 128, 128, false);
  static constexpr uint32_t IDESC_PV = make_idesc(FP8 ? 0u : 1u, 128, D, true);
};

// ---------------------------------------------------------------------------------------
// arithmetic helpers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Packed fp32 pair arithmetic (f32x2, sm_100): one instruction for two lanes of work,
// rounding identical to the scalar forms.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// 2^x on the FMA and integer pipes (software exp2, page "FlashAttention 4 ...", section
// "Αποκορύφωση Λογισμικού μέσω Πυρήνων CUDA"): Cody-Waite split x = j + f with j the nearest
// integer (added to 1.5*2^23 so that rounding leaves j in the low mantissa bits), a cubic
// for 2^f, and j added straight into the exponent field.  x is clamped to >= -125 so the
// result stays a normal float; callers that need exact zeros for -inf select them.
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -125.f);
  const float r = x + 12582912.f;
  const float j = r - 12582912.f;
  const float f = x - j;
  const float q = fmaf(fmaf(fmaf(kE3, f, kE2), f, kE1), f, kE0);
  return __int_as_float(__float_as_int(q) + (__float_as_int(r) << 23));
}

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
  int kvh;        // key/value head (h / group)
  int kvbh;       // key/value head row of batched K/V tensors (b * Hkv + kvh)
  int sq, sk;     // query and key lengths of this item's sequence
  int q_off, k_off;  // first query / key token of the sequence (packed layout; else 0)
  int n;          // number of key tiles visited
  int kt_lo;      // analytic: first key tile
  const uint32_t* entries;  // map: entry list (nullptr for analytic)
};

__device__ __forceinline__ int hi_key(const FwdParams& p, int sk, int ip) {  // last visible key of row i'
  int h = (p.mask_kind & 1) ? ip : ((p.mask_kind & 2) ? ip + p.window - 1 : sk - 1);
  return min(h, sk - 1);
}
__device__ __forceinline__ int lo_key(const FwdParams& p, int ip) {  // first visible key (unclipped)
  return (p.mask_kind & 2) ? ip - p.window + 1 : 0;
}

// Work item at position w of the schedule.  Causal masks (without a window) give the
// 256-row query blocks very different lengths, so they are ordered longest first across
// all heads; otherwise the order is head-major (the K/V of one head stay hot in L2).
__device__ __forceinline__ Item make_item(const FwdParams& p, int w) {
  Item it;
  const int BH = p.B * p.H;   // packed sequences: B is the number of sequences
  if (p.lpt_qb_major) {
    // Longest first within groups of lpt_heads heads, so that the K/V of the heads in
    // flight stay in L2; groups follow one another (the last one may be smaller).
    const int HG = p.lpt_heads > 0 ? p.lpt_heads : BH;
    const int g = w / (HG * p.nqb);
    const int base = g * HG;
    const int hg = min(HG, BH - base);
    const int r = w - base * p.nqb;
    it.qb = p.nqb - 1 - r / hg;
    it.bh = base + r % hg;
  } else {
    it.bh = w / p.nqb;
    it.qb = p.nqb - 1 - w % p.nqb;
  }
  it.b = it.bh / p.H;
  it.h = it.bh % p.H;
  it.kvh = it.h / p.group;
  it.kvbh = it.b * p.Hkv + it.kvh;
  if (p.cu_q != nullptr) {
    it.q_off = __ldg(p.cu_q + it.b);
    it.sq = __ldg(p.cu_q + it.b + 1) - it.q_off;
    it.k_off = __ldg(p.cu_k + it.b);
    it.sk = __ldg(p.cu_k + it.b + 1) - it.k_off;
    // Offsets come from device memory: a sequence outside the tensors or longer than the
    // stated maximum is skipped (nothing loaded or stored) and reported.
    if (it.q_off < 0 || it.sq < 0 || it.sq > p.Sq || it.q_off > p.Tq - it.sq || it.k_off < 0 || it.sk < 0 ||
        it.sk > p.Sk || it.k_off > p.Tk - it.sk) {
      if (it.qb == 0 && it.h == 0) atomicCAS(&g_attn_status, 0, -1 /* ATTN_ERR_INVALID */);
      it.q_off = it.k_off = it.sq = it.sk = 0;
    }
  } else {
    it.q_off = it.k_off = 0;
    it.sq = p.Sq;
    it.sk = p.Sk;
  }
  it.entries = nullptr;
  it.kt_lo = 0;
  if (p.map_counts != nullptr) {
    it.n = p.map_counts[it.b * p.nqb + it.qb];
    it.entries = p.map_entries + (static_cast<size_t>(it.b) * p.nqb + it.qb) * p.nkt;
    return it;
  }
  const int d = it.sk - it.sq;
  int A = it.qb * 256 + d;
  const int Bm = min(it.qb * 256 + 255, it.sq - 1) + d;
  if (p.mask_kind & 1) A = max(A, 0);
  const int klo = max(0, lo_key(p, A));
  const int khi = hi_key(p, it.sk, Bm);
  // a block past the end of its sequence (packed layout) or with no visible key
  if (it.qb * 256 >= it.sq || ((p.mask_kind & 1) && Bm < 0) || khi < klo) {
    it.n = 0;
    return it;
  }
  it.kt_lo = klo / 128;
  it.n = khi / 128 + 1 - it.kt_lo;
  return it;
}

// Static persistent schedule: CTA b takes positions r*G + b (r even) or r*G + G-1-b (r odd),
// r = 0, 1, ...  With the longest-first order this snake keeps the per-CTA totals even.
__device__ __forceinline__ int sched_pos(int r, int b, int G) {
  return r * G + ((r & 1) ? (G - 1 - b) : b);
}

__device__ __forceinline__ int tile_kt(const Item& it, int i) {
  return it.entries ? static_cast<int>(__ldg(it.entries + i) & 0xFFFFFFu) : it.kt_lo + i;
}

// Class of (query tile g, key tile kt): 0 EMPTY, 1 PARTIAL, 2 FULL.
__device__ __forceinline__ int tile_class(const FwdParams& p, const Item& it, int i, int g, int kt) {
  if (it.entries) return static_cast<int>((__ldg(it.entries + i) >> (24 + 2 * g)) & 3u);
  const int r0 = it.qb * 256 + 128 * g;
  if (r0 >= it.sq) return 0;
  const int r1 = min(r0 + 127, it.sq - 1);
  const int d = it.sk - it.sq;
  const int a = r0 + d, bb = r1 + d;
  const int c0 = kt * 128, c1 = c0 + 127, c1v = min(c1, it.sk - 1);
  const bool causal = p.mask_kind & 1, win = p.mask_kind & 2;
  const int i1 = causal ? c0 : (win ? c0 - p.window + 1 : INT_MIN);
  const int i2 = win ? c1v + p.window - 1 : INT_MAX;
  if (max(a, i1) > min(bb, i2)) return 0;
  const bool full = (c1 <= it.sk - 1) && (!win || bb - p.window + 1 <= c0) &&
                    (causal ? (a >= c1) : (!win || a + p.window - 1 >= c1));
  return full ? 2 : 1;
}

// One KV tile of one query tile's online softmax (every thread owns one query row): reads
// the S row from TMEM, applies score_mod and the mask, updates the running max / sum with
// the rescale threshold, writes P over S in TMEM, and rescales O when the max moved.
template <int D, bool FP8, bool SOFTCAP, bool ALIBI>
__device__ __forceinline__ void softmax_tile(const FwdParams& p, const Item& it, int kt, int cls, uint32_t tS,
                                             uint32_t tO, int ip, int jlo_row, int jhi_row, bool has_doc,
                                             int doc_row, float slope_l2, float sq_scale, float v_norm,
                                             float& m_run, float& l_run) {
  using C = Cfg<D, FP8>;
      uint32_t s[128];
      tmem_ld_x128_wait(tS, s);
      float sc = p.scale_log2;     // raw score -> log2 units
      float sc_in = p.sc_in;       // raw score -> tanh argument
      float pv_log2 = 0.f;         // FP8: log2 of the V block's scale relative to v_norm
      float inv_pvf = 1.f;         // and the inverse of that factor
      if constexpr (FP8) {
        const size_t kb = static_cast<size_t>(it.kvbh) * p.nsb_k + kt;
        const float sqk = sq_scale * __ldg(p.k_scale + kb);
        sc *= sqk;
        sc_in *= sqk;
        // P is multiplied by v_scale[kb] / v_norm before its e4m3 rounding; the factor goes
        // into the exponent (one add per tile instead of a multiply per score) and the row
        // sum, which is of the unscaled P, takes its inverse once per tile.
        const float vs = __ldg(p.v_scale + kb);
        pv_log2 = lg2_approx(vs / v_norm);
        inv_pvf = v_norm / vs;
      }
      const int c0 = kt * 128;
      // ---- score_mod (log2 units) and mask; row maximum as a shallow max3 tree.  Each
      //      variant is its own unrolled loop: no runtime branch inside the 128 columns.
      constexpr bool kPlain = !SOFTCAP && !ALIBI;
      float alibi_base = 0.f;
      if constexpr (ALIBI) alibi_base = slope_l2 * static_cast<float>(c0 - ip);
      auto modify = [&](float t, int c) -> float {
        if constexpr (!kPlain) {
          if constexpr (SOFTCAP) {
            // one MUFU tanh per score (PTX bound 2^-10.98 relative; 9.9e-6 measured on B200)
            t = tanh_approx(t * sc_in) * p.sc_out;
            if constexpr (ALIBI) t = fmaf(slope_l2, static_cast<float>(c), t + alibi_base);
          } else if constexpr (ALIBI) {
            // bias first (an FMA with the column as an immediate), then one FMA for the score
            t = fmaf(t, sc, fmaf(slope_l2, static_cast<float>(c), alibi_base));
          }
        }
        return t;
      };
      float mxa[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mxa[u] = kNegInf;
      const bool masked = (cls == 1);
      if (masked) {
        // visible columns of this row: clo <= c <= chi (causal / window / sorted documents),
        // and, for unsorted document ids, doc[c] == doc of the row
        const int clo = jlo_row - c0, chi = jhi_row - c0;
        if (!has_doc) {
          // The row's visible columns as a 128-bit mask (four words), built once per tile;
          // each score then needs one bit test and a select instead of two compares (measured:
          // document masks +14 %, window +4 %).  With ALiBi the compare form measured 2 %
          // faster, so that variant keeps it.
          uint32_t vm[4];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
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
          for (int c = 0; c < 128; c += 2) {
            float t0 = modify(__uint_as_float(s[c]), c);
            float t1 = modify(__uint_as_float(s[c + 1]), c + 1);
            t0 = visible(c) ? t0 : kNegInf;
            t1 = visible(c + 1) ? t1 : kNegInf;
            s[c] = __float_as_uint(t0);
            s[c + 1] = __float_as_uint(t1);
            mxa[(c >> 1) & 7] = fmax3f(mxa[(c >> 1) & 7], t0, t1);
          }
        } else {
          const int* dk = p.doc + static_cast<size_t>(it.b) * p.Sk + c0;
          const int nvalid = p.Sk - c0;
#pragma unroll
          for (int c = 0; c < 128; c += 2) {
            float t0 = modify(__uint_as_float(s[c]), c);
            float t1 = modify(__uint_as_float(s[c + 1]), c + 1);
            const bool v0 = c >= clo && c <= chi && c < nvalid && __ldg(dk + min(c, nvalid - 1)) == doc_row;
            const bool v1 = c + 1 >= clo && c + 1 <= chi && c + 1 < nvalid && __ldg(dk + min(c + 1, nvalid - 1)) == doc_row;
            t0 = v0 ? t0 : kNegInf;
            t1 = v1 ? t1 : kNegInf;
            s[c] = __float_as_uint(t0);
            s[c + 1] = __float_as_uint(t1);
            mxa[(c >> 1) & 7] = fmax3f(mxa[(c >> 1) & 7], t0, t1);
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const float t0 = modify(__uint_as_float(s[c]), c);
          const float t1 = modify(__uint_as_float(s[c + 1]), c + 1);
          if constexpr (!kPlain) {
            s[c] = __float_as_uint(t0);
            s[c + 1] = __float_as_uint(t1);
          }
          mxa[(c >> 1) & 7] = fmax3f(mxa[(c >> 1) & 7], t0, t1);
        }
      }
      float mx = fmax3f(fmax3f(mxa[0], mxa[1], mxa[2]), fmax3f(mxa[3], mxa[4], mxa[5]),
                        fmaxf(mxa[6], mxa[7]));
      // In the plain case the scores are still raw: scale the maximum (scale > 0).
      if constexpr (kPlain) mx = mx * sc;
      // ---- online softmax with the rescale threshold
      bool rescale = false;
      float alpha = 1.f;
      if (mx > m_run + rescale_tau()) {
        if (m_run != kNegInf) {
          alpha = ex2_approx(m_run - mx);
          rescale = true;
          l_run *= alpha;
        }
        m_run = mx;
      }
#ifdef ATTN_ABLATION
      {
        const unsigned r = __ballot_sync(0xffffffffu, rescale), v = __ballot_sync(0xffffffffu, m_run != kNegInf);
        if ((threadIdx.x & 31) == 0) {
          atomicAdd(&g_abl_counts[0], static_cast<unsigned long long>(__popc(r)));
          atomicAdd(&g_abl_counts[1], static_cast<unsigned long long>(__popc(v)));
        }
      }
#endif
      const float msub = (m_run == kNegInf) ? 0.f : m_run;
      // ---- exponentials, packed two per register (f32x2 FMA / ADD), P to TMEM in two halves
      const float2 sc2 = make_float2(sc, sc);
      const float2 nm2 = make_float2(pv_log2 - msub, pv_log2 - msub);
      // 2^a: with kSwExpEvery > 0, one pair in kSwExpEvery goes to the FMA pipes (software
      // exp2); the split depends on the column only, so FULL and PARTIAL tiles agree bit for bit.
      auto pexp = [&](float a, int c) -> float {
        if (kSwExpEvery > 0 && (c >> 1) % kSwDiv == kSwDiv - 1) {
          const float e = exp2_fma(a);
          return masked ? (a == kNegInf ? 0.f : e) : e;
        }
        return ex2_approx(a);
      };
      auto arg2 = [&](int c) -> float2 {
        const float2 v = make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1]));
        if constexpr (kPlain) return ffma2(v, sc2, nm2);
        else return fadd2(v, nm2);
      };
      float2 ls[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) ls[u] = make_float2(0.f, 0.f);
      uint32_t pk[C::P_COLS];
      if constexpr (!FP8) {
#pragma unroll
        for (int c2 = 0; c2 < 64; ++c2) {
          const float2 a = arg2(2 * c2);
          const float2 pp = make_float2(pexp(a.x, 2 * c2), pexp(a.y, 2 * c2 + 1));
          ls[c2 & 3] = fadd2(ls[c2 & 3], pp);
          pk[c2] = pack_bf16x2(pp.x, pp.y);
          if (c2 == 31) tmem_st_x32_nowait<0>(tS, pk);
        }
        tmem_st_x32_wait<32>(tS + 32, pk);
      } else {
#pragma unroll
        for (int c4 = 0; c4 < 32; ++c4) {
          const float2 a = arg2(4 * c4), b = arg2(4 * c4 + 2);
          const float2 p01 = make_float2(pexp(a.x, 4 * c4), pexp(a.y, 4 * c4 + 1));
          const float2 p23 = make_float2(pexp(b.x, 4 * c4 + 2), pexp(b.y, 4 * c4 + 3));
          ls[c4 & 3] = fadd2(ls[c4 & 3], fadd2(p01, p23));
          pk[c4] = pack_e4m3x2(p01.x, p01.y) | (pack_e4m3x2(p23.x, p23.y) << 16);
          if (c4 == 15) tmem_st_x16_nowait<0>(tS, pk);
        }
        tmem_st_x16_wait<16>(tS + 16, pk);
      }
      const float2 l2 = fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3]));
      if constexpr (FP8) l_run += (l2.x + l2.y) * inv_pvf;
      else l_run += l2.x + l2.y;
      // ---- rescale O when the maximum moved by more than TAU (PV_g(i-1) is complete:
      //      its commit preceded the one that signalled S_g(i)).
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          tmem_ld_x32_wait(tO + ch * 32, o);
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st_x32_wait<0>(tO + ch * 32, o);
        }
      }
}

// ---------------------------------------------------------------------------------------
// the kernel (persistent: one CTA per SM walks its share of the work items)
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
            B_PFULL = B_SFULL + 2, B_ODONE = B_PFULL + 2, B_DRAIN = B_ODONE + 2, B_QEMPTY = B_DRAIN + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sptr + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int cta = blockIdx.x;
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
    mbar_init(BAR(B_QEMPTY + 0), 1);
    mbar_init(BAR(B_QEMPTY + 1), 1);
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
  if (warp >= 8) {
    setmaxnreg_dec<kControlRegs>();
  if (warp == kLoadWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const bool varlen = p.cu_q != nullptr;
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      uint32_t lidx = 0;     // ring loads issued (K and V alternate)
      uint32_t qcount = 0;   // Q tile pairs issued
      uint32_t q_issued[2] = {0, 0};   // loads per query buffer: an abort between the two
                                       // buffers of a pair still drains the first
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int w = sched_pos(r, cta, G);
        if (w >= p.num_items) break;
        const Item it = make_item(p, w);
        if (it.n == 0) continue;
        // Query tile g's smem is free once the previous item's last S_g MMA has completed.
        for (int g = 0; g < 2; ++g) {
          if (qcount > 0 && !wait_bounded(BAR(B_QEMPTY + g), (qcount - 1) & 1, abort_flag, tmo)) {
            ok = false;
            break;
          }
          mbar_expect_tx(BAR(B_QFULL + g), C::TILE_BYTES);
          // batched tensors: map (D, S, B*H), coordinates (x, row, b*H+h); packed sequences:
          // map (D, H, T), coordinates (x, h, token)
          const int qrow = it.qb * 256 + 128 * g;
          const int qc1 = varlen ? it.h : qrow, qc2 = varlen ? it.q_off + qrow : it.bh;
          for (int pn = 0; pn < C::NPANEL; ++pn)
            tma_load_3d(sbase + C::OFF_Q + g * C::TILE_BYTES + pn * C::PANEL_BYTES, &tm_q,
                        BAR(B_QFULL + g), pn * C::PANEL_COLS, qc1, qc2, pol_q);
          ++q_issued[g];
        }
        if (!ok) break;
        ++qcount;
        for (int i = 0; i < it.n && ok; ++i) {
          const int kt = tile_kt(it, i);
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t slot = lidx % C::NS;
            if (!wait_bounded(BAR(B_KVEMPTY + slot), ((lidx / C::NS) & 1) ^ 1, abort_flag, tmo)) {
              ok = false;
              break;
            }
            mbar_expect_tx(BAR(B_KVFULL + slot), C::TILE_BYTES);
            const CUtensorMap* tm = kv ? &tm_v : &tm_k;
            const int kc1 = varlen ? it.kvh : kt * 128, kc2 = varlen ? it.k_off + kt * 128 : it.kvbh;
            for (int pn = 0; pn < C::NPANEL; ++pn)
              tma_load_3d(sbase + C::OFF_KV + slot * C::TILE_BYTES + pn * C::PANEL_BYTES, tm,
                          BAR(B_KVFULL + slot), pn * C::PANEL_COLS, kc1, kc2, pol_kv);
            ++lidx;
          }
        }
      }
      // Drain: every copy issued by this thread has landed before the CTA may exit.
      for (int g = 0; g < 2; ++g)
        if (q_issued[g] > 0) drain_bounded(BAR(B_QFULL + g), (q_issued[g] - 1) & 1, tmo);
      for (uint32_t idx = (lidx > C::NS ? lidx - C::NS : 0); idx < lidx; ++idx)
        drain_bounded(BAR(B_KVFULL + idx % C::NS), (idx / C::NS) & 1, tmo);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS[2] = {tbase + C::T_S0, tbase + C::T_S1};
      const uint32_t tO[2] = {tbase + C::T_O0, tbase + C::T_O1};
      // Descriptors of the first tiles; a byte offset b inside the shared window is added as
      // b >> 4 to the start-address field (all addresses stay below 256 KB, so no carry).
      const uint64_t dq = make_sdesc_sw128(sbase + C::OFF_Q, 16, 1024);
      const uint64_t dk = make_sdesc_sw128(sbase + C::OFF_KV, 16, 1024);
      const uint64_t dv = make_sdesc_sw128(sbase + C::OFF_KV, C::PANEL_BYTES, 1024);
      auto qk = [&](int g, uint32_t kslot) {
        const uint64_t a0 = dq + ((g * C::TILE_BYTES) >> 4);
        const uint64_t b0 = dk + ((kslot * C::TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < C::QK_STEPS; ++kk) {
          const int col = kk * C::KSTEP;
          const uint32_t off = ((col / C::PANEL_COLS) * C::PANEL_BYTES + (col % C::PANEL_COLS) * C::EB) >> 4;
          if constexpr (FP8) mma_f8_ss(tS[g], a0 + off, b0 + off, C::IDESC_QK, kk > 0);
          else mma_f16_ss(tS[g], a0 + off, b0 + off, C::IDESC_QK, kk > 0);
        }
      };
      auto pv = [&](int g, uint32_t vslot, bool acc) {
        const uint64_t b0 = dv + ((vslot * C::TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < C::PV_STEPS; ++kk) {
          const uint64_t bd = b0 + ((kk * C::KSTEP * 128) >> 4);
          const uint32_t ta = tS[g] + kk * (C::KSTEP * C::EB / 4);
          if constexpr (FP8) mma_f8_ts(tO[g], ta, bd, C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
          else mma_f16_ts(tO[g], ta, bd, C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
        }
      };
      uint32_t cidx = 0;     // ring loads consumed
      uint32_t tcount = 0;   // tiles processed (phase of s_full / p_full / o_done)
      uint32_t qcount = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int w = sched_pos(r, cta, G);
        if (w >= p.num_items) break;
        const Item it = make_item(p, w);
        if (it.n == 0) continue;
        if (!wait_bounded(BAR(B_QFULL + 0), qcount & 1, abort_flag, tmo) ||
            !wait_bounded(BAR(B_QFULL + 1), qcount & 1, abort_flag, tmo)) {
          ok = false;
          break;
        }
        uint32_t prev_vslot = 0;
        for (int i = 0; i < it.n; ++i) {
          const uint32_t t = tcount + i;
          const uint32_t kidx = cidx + 2 * i, vidx = kidx + 1;
          const uint32_t kslot = kidx % C::NS, vslot = vidx % C::NS;
          // S0(i) = Q0 K_i^T.  It overwrites P0(i-1), which PV0(i-1) (issued earlier by this
          // thread) reads: tcgen05.mma operations from one thread execute in issue order.
          if (!wait_bounded(BAR(B_KVFULL + kslot), (kidx / C::NS) & 1, abort_flag, tmo)) { ok = false; break; }
          tc_fence_after();
          qk(0, kslot);
          mma_commit(BAR(B_SFULL + 0));
          if (i == it.n - 1) mma_commit(BAR(B_QEMPTY + 0));   // last read of Q0 for this item
          // O1 += P1(i-1) V_{i-1}
          if (i > 0) {
            if (!wait_bounded(BAR(B_PFULL + 1), (t - 1) & 1, abort_flag, tmo)) { ok = false; break; }
            tc_fence_after();
            pv(1, prev_vslot, i - 1 > 0);
            mma_commit(BAR(B_ODONE + 1));
            mma_commit(BAR(B_KVEMPTY + prev_vslot));
          }
          // S1(i) = Q1 K_i^T
          qk(1, kslot);
          mma_commit(BAR(B_SFULL + 1));
          mma_commit(BAR(B_KVEMPTY + kslot));
          if (i == it.n - 1) mma_commit(BAR(B_QEMPTY + 1));   // last read of Q1 for this item
          // O0 += P0(i) V_i
          if (!wait_bounded(BAR(B_KVFULL + vslot), (vidx / C::NS) & 1, abort_flag, tmo)) { ok = false; break; }
          if (!wait_bounded(BAR(B_PFULL + 0), t & 1, abort_flag, tmo)) { ok = false; break; }
          tc_fence_after();
          pv(0, vslot, i > 0);
          mma_commit(BAR(B_ODONE + 0));
          prev_vslot = vslot;
        }
        if (!ok) break;
        // O1 += P1(n-1) V_{n-1}
        const uint32_t tl = tcount + it.n - 1;
        if (!wait_bounded(BAR(B_PFULL + 1), tl & 1, abort_flag, tmo)) { ok = false; break; }
        tc_fence_after();
        pv(1, prev_vslot, it.n - 1 > 0);
        mma_commit(BAR(B_ODONE + 1));
        mma_commit(BAR(B_KVEMPTY + prev_vslot));
        cidx += 2 * it.n;
        tcount += it.n;
        ++qcount;
      }
      // Drain: all MMAs issued by this thread are complete before TMEM is freed.
      mma_commit(BAR(B_DRAIN));
      drain_bounded(BAR(B_DRAIN), 0, tmo);
    }
  }
  } else {
    setmaxnreg_inc<kSoftmaxRegs>();
    // ------------------------------------------------------------------ softmax groups
    const int g = warp >> 2;                       // query tile of this group
    const int rloc = (warp & 3) * 32 + lane;       // row within the query tile (= TMEM lane)
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + (g ? C::T_S1 : C::T_S0) + lane_off;
    const uint32_t tO = tbase + (g ? C::T_O1 : C::T_O0) + lane_off;
    const bool has_doc = (p.mask_kind & 4) != 0;
    uint32_t tcount = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int w = sched_pos(r, cta, G);
      if (w >= p.num_items) break;
      const Item it = make_item(p, w);
      const int row = it.qb * 256 + 128 * g + rloc;  // query row within its sequence
      const int ip = row + (it.sk - it.sq);          // bottom-right aligned position
      int jlo_row = lo_key(p, ip);
      int jhi_row = hi_key(p, it.sk, ip);
      const int doc_row = (has_doc && row < p.Sq) ? __ldg(p.doc + static_cast<size_t>(it.b) * p.Sk + row) : 0;
      bool doc_elem = has_doc;   // per-element document test needed on PARTIAL tiles
      if (has_doc && p.doc_sorted != nullptr && __ldg(p.doc_sorted + it.b) != 0) {
        // Non-decreasing ids: the row's document is one run, found by two binary searches,
        // and the visible keys stay one interval.
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
      float sq_scale = 1.f, v_norm = 1.f;
      if constexpr (FP8) {
        const size_t qbase = static_cast<size_t>(it.bh) * p.nsb_q;
        sq_scale = __ldg(p.q_scale + qbase + min(2 * it.qb + g, p.nsb_q - 1));
        const size_t vbase = static_cast<size_t>(it.kvbh) * p.nsb_k;
        float vm = 0.f;
        for (int sb = 0; sb < p.nsb_k; ++sb) vm = fmaxf(vm, __ldg(p.v_scale + vbase + sb));
        v_norm = vm > 0.f ? vm : 1.f;
      }

      float m_run = kNegInf;   // running maximum used for the exponentials (log2 units)
      float l_run = 0.f;       // running row sum against m_run
      for (int i = 0; i < it.n; ++i) {
        const uint32_t t = tcount + i;
        const int kt = tile_kt(it, i);
        const int cls = tile_class(p, it, i, g, kt);
        // The warp-collective TMEM accesses below need every lane to agree on the outcome.
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(B_SFULL + g), t & 1, abort_flag, tmo))) { ok = false; break; }
        tc_fence_after();
        if (cls == 0) {
          // Fully masked for this query tile: P = 0, m and l unchanged.
          uint32_t z[C::P_COLS];
#pragma unroll
          for (int c = 0; c < C::P_COLS; ++c) z[c] = 0u;
          if constexpr (C::P_COLS == 64) tmem_st_x64_wait<0>(tS, z);
          else tmem_st_x32_wait<0>(tS, z);
        } else {
          softmax_tile<D, FP8, SOFTCAP, ALIBI>(p, it, kt, cls, tS, tO, ip, jlo_row, jhi_row, doc_elem,
                                               doc_row, slope_l2, sq_scale, v_norm, m_run, l_run);
        }
        tc_fence_before();
        if (!(p.fault_skip && g == 1 && t == 0)) mbar_arrive(BAR(B_PFULL + g));
      }
      if (!__all_sync(0xffffffffu, ok && !*abort_flag)) {
        ok = false;
        break;
      }
      // ---- epilogue: O / l -> bf16, LSE
      if (it.n > 0) {
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(B_ODONE + g), (tcount + it.n - 1) & 1, abort_flag, tmo))) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      const float inv_l = (l_run > 0.f) ? (v_norm / l_run) : 0.f;
      // batched: O [B, H, Sq, D], LSE [B, H, Sq]; packed: O [Tq, H, D], LSE [H, Tq]
      const bool varlen = p.cu_q != nullptr;
      const size_t orow_idx = varlen ? static_cast<size_t>(it.q_off + row) * p.H + it.h
                                     : static_cast<size_t>(it.bh) * p.Sq + row;
      const size_t lse_idx = varlen ? static_cast<size_t>(it.h) * p.Tq + it.q_off + row
                                    : static_cast<size_t>(it.bh) * p.Sq + row;
      __nv_bfloat16* orow = p.o + orow_idx * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        if (it.n > 0) {
          tmem_ld_x32_wait(tO + ch * 32, o);
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
      if (row < it.sq) {
        const float lse = (l_run > 0.f) ? (m_run + lg2_approx(l_run)) * kLn2 : kNegInf;
        p.lse[lse_idx] = lse;
      }
      tcount += it.n;
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
