// attn_fp4_kernel.cuh — FP4 attention forward with Direct-P, and the MXFP4 quantiser, for
// sm_100a (B200).
//
// The page "Hardware-Aware FP4 FlashAttention-4" (gist.science) describes a forward pass for
// non-causal inference that runs on Blackwell's FP4 tensor cores (summary paragraph), in
// which P is not computed as a probability and then scaled and rounded to FP4: the raw scores
// are mapped straight onto the FP4 codes the tensor cores multiply (Direct-P paragraphs).
// Readings taken here (the page gives no formats):
//   Q, K, V: MXFP4 — e2m1 elements, one power-of-two (E8M0) scale per 32 elements along the
//     contraction axis; V is stored transposed (rows d, keys along the row) so that both
//     products are K-major, which FP4 operands require.
//   P (Direct-P): per row and block of 32 keys, E = floor(max t) - 2 with t the score in log2
//     units; each key's code is the score rounded to the nearest half octave above 2^E,
//     c = clip(rint(2 (t - E) + 2), 0, 7) — two FMAs (one saturating, one rounding down into a
//     constant whose last bits then hold the code), no exponential.
//     The block scale 2^(E - m) (m the row's running reference, an integer) is P's E8M0 scale.
//   O = sum P~ V / sum P~, LSE = ln(sum P~), with P~ the magnitudes the tensor core multiplied.
//
// Both products run as tcgen05.mma kind::mxf4 (block32, E8M0 scales): S = Q K^T with
// M = 128, N = 64, K = 128 (two instructions), O += P V with M = 128, N = 144 (128 of O and 16
// of row sums, below), K = 64 (one).
// Scale factors live in tensor memory; the producer brings them into shared memory in the
// 512-byte layout the tensor core reads (128 rows x 4 scales: byte 16 (r % 32) + 4 (r / 32)
// + block), and the MMA thread copies them with tcgen05.cp (32x128b, replicated to the four
// lane quarters).  P and its scales go through shared memory (FP4 operands come from shared
// memory), P in the 32-byte swizzle layout, one 32-byte row per query row and key tile.  The
// row sum of P~ comes from the tensor core too: 16 rows of e2m1 ones below each stage's V^T make
// the P V product 144 columns wide, column 128 being sum_j P~_j (rescaled with O).
//
// Work item: (b, h, 256 query rows) = two 128-row query groups; key tiles of 64 (S is 64
// columns of tensor memory per group so that both groups' O fit beside it).  Persistent:
// one CTA per SM walks a static share of the items.  12 warps:
//   warps 0-3  softmax group 0 (one thread per query row), warps 4-7 group 1
//   warp  8    producer: Q tiles and scales, then a ring of (128 keys of K, V^T, scales)
//   warp  9    MMA issuer (one thread); allocates and frees tensor memory
//   warps 10-11 idle
// Tensor memory (512 columns): O0 | O1 (144 of 160 each: O and the row sum) | S0 | S1 | scale
// factors.
//
// Every wait is bounded; on time-out the kernel records ATTN_ERR_TIMEOUT, all roles unwind,
// copies and MMAs in flight are drained (bounded), tensor memory is freed.  Nothing traps.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "attn_fwd_kernel.cuh"
#include "ptx.cuh"
#include "tmem_moves.cuh"

namespace attn {
namespace fp4 {

// ---------------------------------------------------------------------------------------
// instruction wrappers (forms as the PTX ISA gives them; no multicast)
// ---------------------------------------------------------------------------------------
// Shared-memory matrix descriptor: bits 0-13 start >> 4, 16-29 leading byte offset >> 4,
// 32-45 stride byte offset >> 4, 46-47 version 1, 61-63 layout (0 none, 6 = 32-byte swizzle,
// 4 = 64-byte swizzle).  K-major swizzled tiles: SBO = 8 rows x row bytes; LBO unused.
constexpr uint32_t kLayoutNone = 0, kLayoutSw32 = 6, kLayoutSw64 = 4;
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(layout) << 61;
  return d;
}

// Instruction descriptor, kind::mxf4 (block-scaled e2m1 x e2m1, both K-major, fp32 D):
//   bits 4-5 B scale byte, 7-9 A format (1 = e2m1), 10-12 B format, 17-22 N >> 3,
//   23 scale format (1 = E8M0), 24-28 M >> 4, 29-30 A scale byte, 31 K (0 = 64).
// The scale bytes pick which bytes of each 32-bit scale column the instruction starts at.
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N, uint32_t sfa_byte, uint32_t sfb_byte) {
  return (sfb_byte << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(M >> 4) << 24) | (sfa_byte << 29);
}

// D[tmem] (+)= (A[smem] x 2^sfa) (B[smem] x 2^sfb)^T, scales from tensor memory.
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// 32 rows x 16 bytes of shared memory -> 4 tensor-memory columns at lanes 0-31, copied to
// all four lane quarters (the scale-factor layout of an M = 128 operand).
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t src_desc) {
#ifdef ATTN_DEBUG_CHECKS
  if (!debug_check((taddr >> 16) == 0u && (taddr & 0xFFFFu) + 4u <= 512u)) return;
#endif
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src_desc) : "memory");
}

// Generic-proxy shared-memory writes become visible to the tensor core's (async proxy) reads.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Two e2m1 codes (round to nearest even, saturating at 6), lo in the low nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// TMA load of one 128-row x 64-byte box (64-byte swizzle); no multicast.
__device__ __forceinline__ void tma_load_box(uint32_t dst, const void* map, uint32_t bar, int c0, int c1, int c2,
                                             uint64_t policy) {
#ifdef ATTN_DEBUG_CHECKS
  if (!debug_check(smem_range_ok(dst, 128u * 64u, 1024u) && c0 >= 0 && (c0 % 16) == 0 && c1 >= 0 && c2 >= 0))
    return;
#endif
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
      "l"(map), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}

// Two fp32 FMAs in one instruction, rounded toward minus infinity.
__device__ __forceinline__ float2 ffma2_rm(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rm.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// 2^e as a float for integer e (0 below the normal range).
__device__ __forceinline__ float exp2i(int e) {
  return e < -126 ? 0.f : __int_as_float((min(e, 127) + 127) << 23);
}

// Byte of the 512-byte scale atom holding row r (0..127) and scale block kb (0..3).
__host__ __device__ constexpr int sf_offset(int r, int kb) { return 16 * (r & 31) + 4 * (r >> 5) + kb; }

// ---------------------------------------------------------------------------------------
// MXFP4 quantiser (HBM-bound).  Rows of 128 elements: x bf16 [BH, S, 128] -> codes
// [BH, S, 64] (element d in byte d / 2, low nibble for even d) and scale atoms
// [BH, ceil(S / 128), 512].  Transposed (V): codes [BH, 128, Sp / 2] with Sp = S rounded up
// to 128 (row d holds the keys; padding keys are zero) and atoms [BH, Sp / 128, 512] indexed
// by (d, key block within the 128 keys).  Scale of a 32-element block: X = floor(log2 amax)
// - 2 (E8M0 byte X + 127; zero block 0); codes = e2m1_rn_satfinite(x * 2^-X).
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ int block_exponent(float amax) {
  const int e = (__float_as_int(amax) >> 23) & 0xFF;      // amax >= 0
  return (amax > 0.f && e > 0) ? max(e - 127 - 2, -127) : -127;
}

__device__ __forceinline__ uint4 encode_block(const float (&v)[32], int X) {
  const float inv = __int_as_float((127 - X) << 23);    // 2^-X, X in [-127, 125]
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t acc = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      acc |= cvt_e2m1x2(v[8 * q + 2 * u] * inv, v[8 * q + 2 * u + 1] * inv) << (8 * u);
    w[q] = acc;
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

constexpr int kQuantRowThreads = 256;

// One thread per (row, 32-element block); rows up to the padded count write their scale
// bytes (0 beyond S) so that every atom is fully defined.
__global__ void __launch_bounds__(kQuantRowThreads)
quant_mxfp4_rows_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ xq, uint8_t* __restrict__ sf,
                        int BH, int S, int nt) {
  const long long gid = static_cast<long long>(blockIdx.x) * kQuantRowThreads + threadIdx.x;
  const long long rows_p = static_cast<long long>(BH) * nt * 128;
  if (gid >= rows_p * 4) return;
  const int kb = static_cast<int>(gid & 3);
  const long long prow = gid >> 2;                 // padded row index over (bh, tile, row)
  const int bh = static_cast<int>(prow / (static_cast<long long>(nt) * 128));
  const int r = static_cast<int>(prow - static_cast<long long>(bh) * nt * 128);
  uint8_t* atom = sf + (static_cast<size_t>(bh) * nt + (r >> 7)) * 512;
  if (r >= S) {
    atom[sf_offset(r & 127, kb)] = 0;
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + (static_cast<size_t>(bh) * S + r) * 128 + 32 * kb);
  float v[32];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = __ldg(src + q);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
      v[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int X = block_exponent(amax);
  reinterpret_cast<uint4*>(xq + (static_cast<size_t>(bh) * S + r) * 64)[kb] = encode_block(v, X);
  atom[sf_offset(r & 127, kb)] = static_cast<uint8_t>(X + 127);
}

// One CTA per (bh, 128-key tile): the 128 x 128 tile goes through shared memory so that each
// thread reads the 32 keys of one (d, key block) down a column.
constexpr int kQuantTThreads = 512;
__global__ void __launch_bounds__(kQuantTThreads)
quant_mxfp4_transposed_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ xq,
                              uint8_t* __restrict__ sf, int S, int nt) {
  __shared__ uint32_t tile[128][65];     // [key][d pair], padded against bank conflicts
  const int bh = blockIdx.x / nt, kt = blockIdx.x % nt;
  const int k0 = kt * 128;
  for (int i = threadIdx.x; i < 128 * 64; i += kQuantTThreads) {
    const int key = i >> 6, dp = i & 63;
    uint32_t w = 0u;
    if (k0 + key < S)
      w = __ldg(reinterpret_cast<const uint32_t*>(x + (static_cast<size_t>(bh) * S + k0 + key) * 128) + dp);
    tile[key][dp] = w;
  }
  __syncthreads();
  const int d = threadIdx.x & 127, kb = threadIdx.x >> 7;
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t w = tile[32 * kb + j][d >> 1];
    v[j] = __uint_as_float((d & 1) ? (w & 0xffff0000u) : (w << 16));
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int X = block_exponent(amax);
  const size_t row_bytes = static_cast<size_t>(nt) * 64;
  reinterpret_cast<uint4*>(xq + (static_cast<size_t>(bh) * 128 + d) * row_bytes + kt * 64)[kb] = encode_block(v, X);
  sf[(static_cast<size_t>(bh) * nt + kt) * 512 + sf_offset(d, kb)] = static_cast<uint8_t>(X + 127);
}

// ---------------------------------------------------------------------------------------
// attention
// ---------------------------------------------------------------------------------------
struct Params {
  __nv_bfloat16* o;     // [B, H, Sq, 128]
  float* lse;           // [B, H, Sq]
  const uint8_t* q_sf;  // [B*H, nqt, 512]
  const uint8_t* k_sf;  // [B*Hkv, nkt, 512]
  const uint8_t* v_sf;  // [B*Hkv, nkt, 512]
  int B, H, Hkv, group, Sq, Sk;
  int nqb, nqt, nkt;    // 256-row query blocks, 128-row query tiles, 128-key tiles
  int num_items;
  float c2;             // 2 * scale * log2(e): raw score -> twice the score in log2 units
  int fault_skip;       // test hook: group 1 skips its first P-ready signal
  unsigned long long timeout_ns;
};

struct Cfg {
  static constexpr int THREADS = 384;
  static constexpr int LOAD_WARP = 8, MMA_WARP = 9;
  static constexpr int TILE = 128 * 64;             // 128 rows of 64 bytes (128 e2m1)
  static constexpr int SF = 512;
  static constexpr int NS = 4;                      // ring of 128-key stages
  static constexpr int OFF_Q = 0;                   // Q0, Q1, then their scale atoms
  static constexpr int OFF_QSF = 2 * TILE;
  static constexpr int OFF_KV = 17 * 1024;
  // K, V^T, then 16 rows of ones below V^T (the row sums as 16 more output columns), scales
  static constexpr int ST_K = 0, ST_V = TILE, ST_ONES = 2 * TILE, ST_KSF = 2 * TILE + 1024, ST_VSF = ST_KSF + SF;
  static constexpr int STAGE = 18 * 1024;
  static constexpr int OFF_P = OFF_KV + NS * STAGE;        // P[g][buf]: 128 rows x 32 bytes
  static constexpr int P_TILE = 128 * 32;
  static constexpr int OFF_PSF = OFF_P + 4 * P_TILE;       // P scale atoms [buf] (both groups)
  static constexpr int OFF_ONESF = OFF_PSF + 2 * SF;      // scale atom of the ones rows (all 2^0)
  static constexpr int OFF_BAR = OFF_ONESF + SF;
  // barriers: QFULL 2, QEMPTY 2, KVFULL NS, KVEMPTY NS, SFULL, SFREE (both groups), PFULL 2, PFREE 2,
  // DRAIN 1.  PFULL[b] / PFREE[b] serve both groups: P of tile k (buffer k & 1) of both groups
  // is ready / both P V products of tile k are complete.  "P V of tile k is complete" is read
  // from PFREE[k & 1]: the softmax waited for that barrier's previous phase before writing P of
  // tile k, so the parity it waits for next is never ambiguous.
  static constexpr int B_QFULL = 0, B_QEMPTY = 2, B_KVFULL = 4, B_KVEMPTY = 4 + NS, B_SFULL = 4 + 2 * NS,
                       B_SFREE = B_SFULL + 2, B_PFULL = B_SFREE + 2, B_PFREE = B_PFULL + 2,
                       B_DRAIN = B_PFREE + 2, NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int ON = 144;                          // O columns per group: 128 of O, then the row sum
  static constexpr uint32_t O_STRIDE = 160;               // group 1's O (32-column aligned)
  static constexpr uint32_t T_O = 0, T_S = 2 * O_STRIDE, T_SFQ = T_S + 128, T_SFP = T_SFQ + 8, T_SFK = T_SFP + 8,
                            T_SFV = T_SFK + 4 * NS;            // V^T scales: 8 columns per stage (4 + the ones')
  static constexpr float kTau = 8.f;                 // rescale threshold (octaves)
  static constexpr float kMagic = 12582912.f;        // 1.5 * 2^23: the unit of its last bit is 1
};
static_assert(Cfg::OFF_KV >= Cfg::OFF_QSF + 2 * Cfg::SF, "Q region overlaps the ring");
static_assert(Cfg::SMEM_BYTES <= 227 * 1024, "shared memory");
static_assert(Cfg::T_SFV + 8 * Cfg::NS <= Cfg::TMEM_COLS, "tensor memory");

__device__ __forceinline__ void item_of(const Params& p, int w, int& bh, int& qb, int& kvbh) {
  bh = w / p.nqb;
  qb = w % p.nqb;
  const int b = bh / p.H, h = bh % p.H;
  kvbh = b * p.Hkv + h / p.group;
}

__global__ void __launch_bounds__(Cfg::THREADS, 1)
attn_fp4_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_vt, const Params p) {
  using C = Cfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sptr = smem_raw + (sbase - raw);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sptr + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int cta = blockIdx.x;
  const unsigned long long tmo = p.timeout_ns;
  const int n_sub = 2 * p.nkt;   // 64-key tiles per item

  if (threadIdx.x == 0) {
    for (int g = 0; g < 2; ++g) {
      mbar_init(BAR(C::B_QFULL + g), 1);
      mbar_init(BAR(C::B_QEMPTY + g), 1);
      if (g == 0) {
        mbar_init(BAR(C::B_SFULL), 1);     // both groups' S of one tile computed
        mbar_init(BAR(C::B_SFREE), 8);     // both groups have read their S (one arrival per softmax warp)
      }
      for (int b = 0; b < 2; ++b) {
        if (g == 0) {
          mbar_init(BAR(C::B_PFULL + b), 8);     // both groups' P of one tile (one arrival per softmax warp)
          mbar_init(BAR(C::B_PFREE + b), 1);     // both groups' P V of that tile complete
        }
      }
    }
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(BAR(C::B_KVFULL + s), 1);
      mbar_init(BAR(C::B_KVEMPTY + s), 1);
    }
    mbar_init(BAR(C::B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // 16 rows of e2m1 ones (code 2) below each stage's V^T tile, and a scale atom of 2^0: the
  // P V product then also sums P~ over the keys (output columns 128..143 of each group)
  for (int i = threadIdx.x; i < C::NS * 256; i += C::THREADS)
    reinterpret_cast<uint32_t*>(sptr + C::OFF_KV + (i >> 8) * C::STAGE + C::ST_ONES)[i & 255] = 0x22222222u;
  for (int i = threadIdx.x; i < C::SF / 4; i += C::THREADS)
    reinterpret_cast<uint32_t*>(sptr + C::OFF_ONESF)[i] = 0x7F7F7F7Fu;
  fence_proxy_async_smem();
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::LOAD_WARP && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_vt);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  if (warp == C::LOAD_WARP) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      uint32_t lidx = 0, qcount = 0;
      uint32_t q_issued[2] = {0, 0};
      bool ok = true;
      for (int w = cta; ok && w < p.num_items; w += G) {
        int bh, qb, kvbh;
        item_of(p, w, bh, qb, kvbh);
        for (int g = 0; g < 2; ++g) {
          if (qcount > 0 && !wait_bounded(BAR(C::B_QEMPTY + g), (qcount - 1) & 1, abort_flag, tmo)) {
            ok = false;
            break;
          }
          mbar_expect_tx(BAR(C::B_QFULL + g), C::TILE + C::SF);
          tma_load_box(sbase + C::OFF_Q + g * C::TILE, &tm_q, BAR(C::B_QFULL + g), 0, qb * 256 + 128 * g, bh, pol_q);
          const int qt = min(2 * qb + g, p.nqt - 1);
          bulk_load(sbase + C::OFF_QSF + g * C::SF, p.q_sf + (static_cast<size_t>(bh) * p.nqt + qt) * C::SF, C::SF,
                    BAR(C::B_QFULL + g));
          ++q_issued[g];
        }
        if (!ok) break;
        ++qcount;
        for (int kt = 0; kt < p.nkt; ++kt) {
          const uint32_t slot = lidx % C::NS;
          if (!wait_bounded(BAR(C::B_KVEMPTY + slot), ((lidx / C::NS) & 1) ^ 1, abort_flag, tmo)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + C::OFF_KV + slot * C::STAGE;
          const uint32_t bar = BAR(C::B_KVFULL + slot);
          mbar_expect_tx(bar, 2 * C::TILE + 2 * C::SF);
          tma_load_box(st + C::ST_K, &tm_k, bar, 0, kt * 128, kvbh, pol_kv);
          tma_load_box(st + C::ST_V, &tm_vt, bar, kt * 64, 0, kvbh, pol_kv);
          const size_t a = (static_cast<size_t>(kvbh) * p.nkt + kt) * C::SF;
          bulk_load(st + C::ST_KSF, p.k_sf + a, C::SF, bar);
          bulk_load(st + C::ST_VSF, p.v_sf + a, C::SF, bar);
          ++lidx;
        }
      }
      for (int g = 0; g < 2; ++g)
        if (q_issued[g] > 0) drain_bounded(BAR(C::B_QFULL + g), (q_issued[g] - 1) & 1, tmo);
      for (uint32_t idx = (lidx > C::NS ? lidx - C::NS : 0); idx < lidx; ++idx)
        drain_bounded(BAR(C::B_KVFULL + idx % C::NS), (idx / C::NS) & 1, tmo);
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tO[2] = {tbase + C::T_O, tbase + C::T_O + C::O_STRIDE};
      const uint32_t tS[2] = {tbase + C::T_S, tbase + C::T_S + 64};
      const uint32_t tSFQ[2] = {tbase + C::T_SFQ, tbase + C::T_SFQ + 4};
      auto sfdesc = [&](uint32_t addr) { return sdesc(addr, 16, 128, kLayoutNone); };
      // the ones rows' scales (2^0) sit in column 4 of every stage's V^T scale columns for good
      for (int s = 0; s < C::NS; ++s) tmem_cp_sf(tbase + C::T_SFV + 8 * s + 4, sfdesc(sbase + C::OFF_ONESF));
      uint32_t tc = 0, cidx = 0, qcount = 0;
      bool ok = true;
      for (int w = cta; ok && w < p.num_items; w += G) {
        if (!wait_bounded(BAR(C::B_QFULL + 0), qcount & 1, abort_flag, tmo) ||
            !wait_bounded(BAR(C::B_QFULL + 1), qcount & 1, abort_flag, tmo)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int g = 0; g < 2; ++g) tmem_cp_sf(tSFQ[g], sfdesc(sbase + C::OFF_QSF + g * C::SF));
        for (int j = 0; j <= n_sub && ok; ++j) {
          if (j < n_sub) {
            const uint32_t stage = cidx + (j >> 1), slot = stage % C::NS;
            const uint32_t st = sbase + C::OFF_KV + slot * C::STAGE;
            if ((j & 1) == 0) {
              if (!wait_bounded(BAR(C::B_KVFULL + slot), (stage / C::NS) & 1, abort_flag, tmo)) { ok = false; break; }
              tc_fence_after();
              tmem_cp_sf(tbase + C::T_SFK + 4 * slot, sfdesc(st + C::ST_KSF));
              tmem_cp_sf(tbase + C::T_SFV + 8 * slot, sfdesc(st + C::ST_VSF));
            }
            const uint32_t t = tc + j;
            // S0 and S1 are free once both groups' threads have read the previous tile's scores.
            if (t >= 1 && !wait_bounded(BAR(C::B_SFREE), (t - 1) & 1, abort_flag, tmo)) { ok = false; break; }
            tc_fence_after();
            for (int g = 0; g < 2; ++g) {
#pragma unroll
              for (int kk = 0; kk < 2; ++kk) {
                const uint64_t a = sdesc(sbase + C::OFF_Q + g * C::TILE + 32 * kk, 16, 512, kLayoutSw64);
                const uint64_t b = sdesc(st + C::ST_K + (j & 1) * 64 * 64 + 32 * kk, 16, 512, kLayoutSw64);
                mma_mxf4(tS[g], a, b, idesc_mxf4(128, 64, 2 * kk, 2 * kk), tSFQ[g],
                         tbase + C::T_SFK + 4 * slot + 2 * (j & 1), kk > 0);
              }
              if (j == n_sub - 1) mma_commit(BAR(C::B_QEMPTY + g));   // last read of Q_g
            }
            mma_commit(BAR(C::B_SFULL));
            if (!ok) break;
          }
          if (j >= 1) {
            const int jp = j - 1;
            const uint32_t tp = tc + jp, buf = tp & 1;
            const uint32_t stage = cidx + (jp >> 1), slot = stage % C::NS;
            const uint32_t st = sbase + C::OFF_KV + slot * C::STAGE;
            // both groups' P scales share one atom (group g in bytes 2g, 2g + 1 of each row):
            // one copy to tensor memory serves both products
            if (!wait_bounded(BAR(C::B_PFULL + buf), (tp >> 1) & 1, abort_flag, tmo)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t tsfp = tbase + C::T_SFP + 4 * buf;
            tmem_cp_sf(tsfp, sfdesc(sbase + C::OFF_PSF + buf * C::SF));
            for (int g = 0; g < 2; ++g) {
              const uint64_t a = sdesc(sbase + C::OFF_P + (2 * g + buf) * C::P_TILE, 16, 256, kLayoutSw32);
              const uint64_t b = sdesc(st + C::ST_V + 32 * (jp & 1), 16, 512, kLayoutSw64);
              mma_mxf4(tO[g], a, b, idesc_mxf4(128, C::ON, 2 * g, 2 * (jp & 1)), tsfp, tbase + C::T_SFV + 8 * slot,
                       jp > 0 ? 1u : 0u);
            }
            mma_commit(BAR(C::B_PFREE + buf));
            if (!ok) break;
            if (jp & 1) mma_commit(BAR(C::B_KVEMPTY + slot));
          }
        }
        if (!ok) break;
        cidx += p.nkt;
        tc += n_sub;
        ++qcount;
      }
      mma_commit(BAR(C::B_DRAIN));
      drain_bounded(BAR(C::B_DRAIN), 0, tmo);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax (Direct-P)
    const int g = warp >> 2;
    const int rloc = (warp & 3) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + C::T_S + 64 * g + lane_off;
    const uint32_t tO = tbase + C::T_O + C::O_STRIDE * g + lane_off;   // O, then the row sum at column 128
    const float c2 = p.c2;
    constexpr float kNegInfF = -__builtin_huge_valf();
    // P row (32 bytes) of this thread in the 32-byte swizzle: chunk c at c ^ bit 2 of the row
    const uint32_t prow_off = (rloc >> 3) * 256 + (rloc & 7) * 32;
    const uint32_t psw = (rloc >> 2) & 1;
    const uint32_t psf_off = sf_offset(rloc, 2 * g);
    uint32_t tc = 0;
    bool ok = true;
    for (int w = cta; ok && w < p.num_items; w += G) {
      int bh, qb, kvbh;
      item_of(p, w, bh, qb, kvbh);
      const int row = qb * 256 + 128 * g + rloc;
      float m = kNegInfF;     // running reference (an integer, log2 units)
      for (int j = 0; j < n_sub; ++j) {
        const uint32_t t = tc + j, buf = t & 1;
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_SFULL), t & 1, abort_flag, tmo))) { ok = false; break; }
        tc_fence_after();
        uint32_t s[64];
        tmem_ld_x64_wait(tS, s);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_SFREE));
        // keys past the end of the sequence take no part
        const int nvalid = p.Sk - 64 * j;
        if (nvalid < 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= nvalid) s[c] = __float_as_uint(kNegInfF);
        }
        float bm[2];
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          float a[4] = {kNegInfF, kNegInfF, kNegInfF, kNegInfF};
#pragma unroll
          for (int c = 0; c < 32; c += 8)
#pragma unroll
            for (int u = 0; u < 4; ++u)
              a[u] = fmax3f(a[u], __uint_as_float(s[32 * blk + c + 2 * u]), __uint_as_float(s[32 * blk + c + 2 * u + 1]));
          bm[blk] = fmax3f(a[0], a[1], fmaxf(a[2], a[3]));
        }
        // block exponents E = floor(max t) - 2 (t = s * c2 / 2), the row reference m
        float E[2];
        bool live[2];
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          live[blk] = bm[blk] != kNegInfF;
          E[blk] = live[blk] ? floorf(bm[blk] * (0.5f * c2)) - 2.f : kNegInfF;
        }
        const float mt = fmaxf(E[0], E[1]) + 2.f;
        bool rescale = false;
        float alpha = 1.f;
        if (mt > m + C::kTau) {
          if (m != kNegInfF) {
            alpha = exp2i(static_cast<int>(m - mt));
            rescale = true;
          }
          m = mt;
        }
        // codes: with y2 = 2 (t - E) + 2, z = sat((y2 + 1/2) / 8) (one FMA with saturation) and
        // code = floor((8 - 2^-21) z), which is rint(y2) clipped to [0, 7] away from exact ties;
        // the floor is a round-down FMA into 1.5 * 2^23, whose last bits then hold the code.
        uint32_t pw[8];
        uint32_t sfb = 0;
        const float a8 = 0.125f * c2;
        const float2 k8 = make_float2(7.99999952f, 7.99999952f), mg = make_float2(C::kMagic, C::kMagic);
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          const int e = live[blk] ? static_cast<int>(E[blk] - m) : -1000;   // scale exponent
          const bool use = e >= -127;
          const float b8 = use ? (2.5f - 2.f * E[blk]) * 0.125f : kNegInfF;
          sfb |= static_cast<uint32_t>(use ? e + 127 : 0) << (8 * blk);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t byte[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int c = 32 * blk + 8 * q + 2 * u;
              const float z0 = __saturatef(fmaf(__uint_as_float(s[c]), a8, b8));
              const float z1 = __saturatef(fmaf(__uint_as_float(s[c + 1]), a8, b8));
              const float2 r = ffma2_rm(make_float2(z0, z1), k8, mg);
              // low byte: code1 << 4 | code0 (the constant's low byte is zero)
              byte[u] = (__float_as_uint(r.y) << 4) + __float_as_uint(r.x);
            }
            const uint32_t wv = __byte_perm(__byte_perm(byte[0], byte[1], 0x0040), __byte_perm(byte[2], byte[3], 0x0040),
                                            0x5410);
            pw[4 * blk + q] = wv;
          }
        }
        // P and its scales to shared memory (buffer buf is free once PV of tile t-2 is done)
        if (t >= 2 && !__all_sync(0xffffffffu, wait_bounded(BAR(C::B_PFREE + buf), ((t >> 1) - 1) & 1,
                                                            abort_flag, tmo))) {
          ok = false;
          break;
        }
        uint8_t* prow = sptr + C::OFF_P + (2 * g + buf) * C::P_TILE + prow_off;
        *reinterpret_cast<uint4*>(prow + (psw << 4)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        *reinterpret_cast<uint4*>(prow + ((psw ^ 1u) << 4)) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
        *reinterpret_cast<uint16_t*>(sptr + C::OFF_PSF + buf * C::SF + psf_off) =
            static_cast<uint16_t>(sfb);
        fence_proxy_async_smem();
        // rescale O when the reference moved (PV of tile t-1 has completed first)
        if (__any_sync(0xffffffffu, rescale)) {
          if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_PFREE + ((t - 1) & 1)), ((t - 1) >> 1) & 1,
                                                    abort_flag, tmo))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t o[32];
            tmem_ld_x32_wait(tO + ch * 32, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st_x32_wait<0>(tO + ch * 32, o);
          }
          uint32_t ls[16];   // the row sum columns
          tmem_ld_x16_wait(tO + 128, ls);
#pragma unroll
          for (int c = 0; c < 16; ++c) ls[c] = __float_as_uint(__uint_as_float(ls[c]) * alpha);
          tmem_st_x16_wait<0>(tO + 128, ls);
        }
        tc_fence_before();
        // one arrival per warp: the warp's stores and fences above come first
        __syncwarp();
        if (lane == 0 && !(p.fault_skip && g == 1 && t == 0)) mbar_arrive(BAR(C::B_PFULL + buf));
      }
      if (!__all_sync(0xffffffffu, ok && !*abort_flag)) {
        ok = false;
        break;
      }
      // ---- epilogue: O / l -> bf16, LSE
      const uint32_t last = tc + n_sub - 1;
      if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_PFREE + (last & 1)), (last >> 1) & 1, abort_flag,
                                                tmo))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t ls[16];
      tmem_ld_x16_wait(tO + 128, ls);
      const float l = __uint_as_float(ls[0]);   // sum of P~ against 2^m, from the tensor core
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.Sq + row) * 128;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t o[32];
        tmem_ld_x32_wait(tO + ch * 32, o);
        uint32_t wv[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          wv[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
        if (row < p.Sq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) __stcs(dst + v, make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]));
        }
      }
      if (row < p.Sq)
        p.lse[static_cast<size_t>(bh) * p.Sq + row] = l > 0.f ? (m + lg2_approx(l)) * kLn2 : kNegInf;
      tc += n_sub;
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace fp4
}  // namespace attn
