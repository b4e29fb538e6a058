// attn_api.cu — host side of libattn.so: argument checks, TMA tensor-map encoding, kernel
// selection and launch, the stream-ordered workspace, the device status word.
//
// The C-ABI is declared (with its contract) in include/attn.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#ifdef ATTN_ABLATION
#include "attn_ablation.h"
#endif
#include "attn_bwd_kernel.cuh"
#include "attn_fwd_kernel.cuh"
#include "attn_fp4_kernel.cuh"
#include "attn_fwd_pair_kernel.cuh"
#include "quant_kernel.cuh"
#include "tile_map_kernel.cuh"

namespace {

using attn::FwdParams;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool init = false;
  bool supported = false;
  int sms = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::atomic<int> g_fault_skip{0};
std::atomic<int> g_timeout_ms{1000};

int current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[*dev];
  if (!d.init) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    d.supported = (major == 10 && minor == 0);
    d.sms = sms;
    d.init = true;
  }
  if (!d.supported) return ATTN_ERR_UNSUPPORTED;
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return ATTN_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks shared by the attention entry points (host only; nothing is launched on failure).
int check_common(const void* q, const void* k, const void* v, const void* o, const void* lse,
                 int B, int H, int Sq, int Sk, int D, float scale, int mask_kind, int window,
                 float softcap, const float* alibi, const int* doc_ids) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_INVALID;
  if (alibi && !aligned16(alibi)) return ATTN_ERR_INVALID;
  if (doc_ids && !aligned16(doc_ids)) return ATTN_ERR_INVALID;
  if (D != 64 && D != 128) return ATTN_ERR_INVALID;
  if (B <= 0 || H <= 0 || Sq <= 0 || Sk <= 0) return ATTN_ERR_INVALID;
  if (Sq > ATTN_MAX_SEQ || Sk > ATTN_MAX_SEQ) return ATTN_ERR_INVALID;
  if (static_cast<long long>(B) * H * ((Sq + 255) / 256) > 0x7fffffffLL) return ATTN_ERR_INVALID;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID;
  if (mask_kind & ~(ATTN_MASK_CAUSAL | ATTN_MASK_WINDOW | ATTN_MASK_DOC)) return ATTN_ERR_INVALID;
  if ((mask_kind & ATTN_MASK_WINDOW) && window <= 0) return ATTN_ERR_INVALID;
  if ((mask_kind & ATTN_MASK_DOC) && (doc_ids == nullptr || Sq != Sk)) return ATTN_ERR_INVALID;
  if (!std::isfinite(softcap)) return ATTN_ERR_INVALID;
  return ATTN_OK;
}

// Packed token-major tensor [T, Hx, D]: map (D, Hx, T), box 64 or 128 columns x 1 head x
// 128 tokens, so a box lands in shared memory exactly as a batched tile does.
int encode_map_thd(CUtensorMap* map, const void* ptr, int Hx, int T, int D, int box_tokens = 128) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hx), static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(Hx) * D * 2};
  cuuint32_t box[3] = {64u, 1u, static_cast<cuuint32_t>(box_tokens)};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

int encode_map(CUtensorMap* map, const void* ptr, bool fp8, int BH, int S, int D, int box_rows = 128) {
  const int eb = fp8 ? 1 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * eb, static_cast<cuuint64_t>(S) * D * eb};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / eb), static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = g_encode(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                              const_cast<void*>(ptr), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool FP8, bool SOFTCAP, bool ALIBI>
int launch_fwd_t(int dev, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                 const FwdParams& p, cudaStream_t stream) {
  using C = attn::Cfg<D, FP8>;
  auto kern = attn::attn_fwd_kernel<D, FP8, SOFTCAP, ALIBI>;
  static bool attr_set[kMaxDevices] = {};
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return ATTN_ERR_CUDA;
    attr_set[dev] = true;
  }
  // Persistent grid: one CTA per SM (the kernel holds all 512 TMEM columns and most of
  // shared memory, so only one CTA fits on an SM anyway), never more CTAs than work items.
  const int grid = p.num_items < g_dev[dev].sms ? p.num_items : g_dev[dev].sms;
  kern<<<static_cast<unsigned>(grid), attn::kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool FP8>
int launch_fwd_d(int dev, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                 const FwdParams& p, bool softcap, bool alibi, cudaStream_t s) {
  if (softcap) {
    return alibi ? launch_fwd_t<D, FP8, true, true>(dev, tq, tk, tv, p, s)
                 : launch_fwd_t<D, FP8, true, false>(dev, tq, tk, tv, p, s);
  }
  return alibi ? launch_fwd_t<D, FP8, false, true>(dev, tq, tk, tv, p, s)
               : launch_fwd_t<D, FP8, false, false>(dev, tq, tk, tv, p, s);
}

// The pair kernel (attn_fwd_pair_kernel, BF16, D = 128) runs through attn_fwd_pair only:
// measured on B200 it reaches about 80 % of the single-CTA kernel's rate (causal B4 H16 S4096
// 738 against 925 TFLOP/s, non-causal B1 H32 S32768 885 against 1055), so the other entry
// points keep the single-CTA kernel.  ATTN_PAIR_SPLIT softmax warps share each query row (2:
// 64 keys each; 4 measured slower).
#ifndef ATTN_PAIR_SPLIT
#define ATTN_PAIR_SPLIT 2
#endif

template <bool SOFTCAP, bool ALIBI>
int launch_pair_t(int dev, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                  cudaStream_t stream) {
  using C = attn::CfgPair<ATTN_PAIR_SPLIT>;
  auto kern = attn::attn_fwd_pair_kernel<ATTN_PAIR_SPLIT, SOFTCAP, ALIBI>;
  static bool attr_set[kMaxDevices] = {};
  static int clusters[kMaxDevices] = {};
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return ATTN_ERR_CUDA;
    attr_set[dev] = true;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (clusters[dev] == 0) {
    // Persistent grid: as many pairs as can be resident at once (one CTA per SM; SMs that
    // cannot be paired inside their GPC stay idle).
    cfg.gridDim = dim3(static_cast<unsigned>(2 * (g_dev[dev].sms / 2)), 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) return ATTN_ERR_CUDA;
    clusters[dev] = n;
  }
  const int pairs = p.num_items < clusters[dev] ? p.num_items : clusters[dev];
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p) != cudaSuccess) return ATTN_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int launch_pair(int dev, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                bool softcap, bool alibi, cudaStream_t s) {
  if (softcap) {
    return alibi ? launch_pair_t<true, true>(dev, tq, tk, tv, p, s) : launch_pair_t<true, false>(dev, tq, tk, tv, p, s);
  }
  return alibi ? launch_pair_t<false, true>(dev, tq, tk, tv, p, s) : launch_pair_t<false, false>(dev, tq, tk, tv, p, s);
}

// Fills the parameter block shared by the BF16 and FP8 paths.
FwdParams make_params(void* o, float* lse, int B, int H, int Hkv, int Sq, int Sk, float scale, int mask_kind,
                      int window, float softcap, const float* alibi, const int* doc_ids) {
  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.group = H / Hkv;
  p.Sq = Sq;
  p.Sk = Sk;
  p.nqb = (Sq + 255) / 256;
  p.nkt = (Sk + 127) / 128;
  p.mask_kind = mask_kind;
  // A window at least Sq + Sk wide removes nothing; clamping keeps the index math in int32.
  const long long wmax = static_cast<long long>(Sq) + Sk;
  p.window = (mask_kind & ATTN_MASK_WINDOW) ? static_cast<int>(window < wmax ? window : wmax) : 0;
  const double log2e = 1.4426950408889634;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * log2e);
  if (softcap > 0.f) {
    p.sc_in = static_cast<float>(static_cast<double>(scale) / softcap);
    p.sc_out = static_cast<float>(static_cast<double>(softcap) * log2e);
  }
  p.alibi = alibi;
  p.doc = (mask_kind & ATTN_MASK_DOC) ? doc_ids : nullptr;
  const long long items = static_cast<long long>(B) * H * p.nqb;
  p.num_items = static_cast<int>(items);
  // Causal without a window: query blocks differ a lot in length -> longest first.
  p.lpt_qb_major = ((mask_kind & ATTN_MASK_CAUSAL) && !(mask_kind & (ATTN_MASK_WINDOW | ATTN_MASK_DOC))) ? 1 : 0;
  p.lpt_heads = 0;
  p.fault_skip = g_fault_skip.load();
  p.timeout_ns = static_cast<unsigned long long>(g_timeout_ms.load()) * 1000000ull;
  return p;
}

#ifndef ATTN_L2_GROUP_BYTES
#define ATTN_L2_GROUP_BYTES 0
#endif
// Causal longest-first order can work through groups of heads whose K and V together take at
// most ATTN_L2_GROUP_BYTES, so that the K/V tiles the CTAs in flight re-read come from L2.
// Measured on B200 with 32 MB groups it was much slower (causal B4 H16 S4096: 940 -> 712
// TFLOP/s; FP8 causal 1101 -> 1004; grouped-query 1002 -> 914): the per-group longest-first
// order leaves the CTAs' totals uneven.  0 (the default) keeps one group over all heads.
int lpt_head_group(const FwdParams& p, int Sk, int D, int eb) {
  if (!p.lpt_qb_major || ATTN_L2_GROUP_BYTES <= 0) return 0;
  const long long kv_head = 2ll * Sk * D * eb;
  long long kv_heads = ATTN_L2_GROUP_BYTES / (kv_head > 0 ? kv_head : 1);
  if (kv_heads < 1) kv_heads = 1;
  long long heads = kv_heads * p.group;          // query heads per group
  const long long BH = static_cast<long long>(p.B) * p.H;
  return heads >= BH ? 0 : static_cast<int>(heads);
}

int launch_tile_map(int* counts, uint32_t* entries, int B, int Sq, int Sk, int mask_kind, int window,
                    const int* doc_ids, cudaStream_t stream, int* sorted_flags = nullptr) {
  const int nqb = (Sq + 255) / 256, nkt = (Sk + 127) / 128;
  const long long wmax = static_cast<long long>(Sq) + Sk;
  const int w = (mask_kind & ATTN_MASK_WINDOW) ? static_cast<int>(window < wmax ? window : wmax) : 0;
  dim3 grid(nqb, B);
  attn::tile_map_kernel<<<grid, attn::kMapThreads, 0, stream>>>(counts, entries, Sq, Sk, mask_kind, w,
                                                                 (mask_kind & ATTN_MASK_DOC) ? doc_ids : nullptr,
                                                                 nqb, nkt, sorted_flags);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Workspace of the document path: counts [B*nqb] | entries [B*nqb*nkt] | sorted flags [B],
// each part 16-byte aligned.
size_t ws_counts_bytes(int B, int Sq) { return ((static_cast<size_t>(B) * ((Sq + 255) / 256) * sizeof(int) + 15) & ~size_t(15)); }
size_t ws_entries_bytes(int B, int Sq, int Sk) {
  return ((static_cast<size_t>(B) * ((Sq + 255) / 256) * ((Sk + 127) / 128) * sizeof(uint32_t) + 15) & ~size_t(15));
}
size_t ws_bytes_for_map(int B, int Sq, int Sk) {
  return ws_counts_bytes(B, Sq) + ws_entries_bytes(B, Sq, Sk) + static_cast<size_t>(B) * sizeof(int);
}

// Shared body of attn_fwd / attn_fwd_with_map / attn_fwd_fp8.
int run_fwd(bool fp8, const void* q, const void* k, const void* v, const float* qs, const float* ks,
            const float* vs, void* o, float* lse, int B, int H, int Hkv, int Sq, int Sk, int D, float scale,
            int mask_kind, int window, float softcap, const float* alibi, const int* doc_ids,
            const int* counts, const uint32_t* entries, cudaStream_t stream, bool pair = false) {
  int rc = check_common(q, k, v, o, lse, B, H, Sq, Sk, D, scale, mask_kind, window, softcap, alibi, doc_ids);
  if (rc != ATTN_OK) return rc;
  if (Hkv <= 0 || H % Hkv != 0) return ATTN_ERR_INVALID;
  if (fp8 && (D != 128 || !qs || !ks || !vs)) return ATTN_ERR_INVALID;
  if (pair && (fp8 || D != 128)) return ATTN_ERR_INVALID;
  if ((counts == nullptr) != (entries == nullptr)) return ATTN_ERR_INVALID;
  // the tile-map build launches one grid row per batch entry (grid.y <= 65535)
  if (counts == nullptr && (mask_kind & ATTN_MASK_DOC) && B > 65535) return ATTN_ERR_INVALID;
  int dev = 0;
  if ((rc = current_device(&dev)) != ATTN_OK) return rc;

  FwdParams p = make_params(o, lse, B, H, Hkv, Sq, Sk, scale, mask_kind, window, softcap, alibi, doc_ids);
  if (fp8) {
    p.q_scale = qs;
    p.k_scale = ks;
    p.v_scale = vs;
    p.nsb_q = (Sq + 127) / 128;
    p.nsb_k = (Sk + 127) / 128;
  }
  p.lpt_heads = lpt_head_group(p, Sk, D, fp8 ? 1 : 2);
  CUtensorMap tq, tk, tv;
  if (encode_map(&tq, q, fp8, B * H, Sq, D) != ATTN_OK ||
      encode_map(&tk, k, fp8, B * Hkv, Sk, D, pair ? 64 : 128) != ATTN_OK ||
      encode_map(&tv, v, fp8, B * Hkv, Sk, D) != ATTN_OK)
    return ATTN_ERR_CUDA;

  void* ws = nullptr;
  if (counts == nullptr && (mask_kind & ATTN_MASK_DOC)) {
    // Document masks need the tile map: a stream-ordered workspace for this call.
    if (cudaMallocAsync(&ws, ws_bytes_for_map(B, Sq, Sk), stream) != cudaSuccess) return ATTN_ERR_NOMEM;
    int* c = static_cast<int*>(ws);
    uint32_t* e = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + ws_counts_bytes(B, Sq));
    int* sorted = reinterpret_cast<int*>(static_cast<char*>(ws) + ws_counts_bytes(B, Sq) + ws_entries_bytes(B, Sq, Sk));
    rc = launch_tile_map(c, e, B, Sq, Sk, mask_kind, window, doc_ids, stream, sorted);
    p.doc_sorted = sorted;
    if (rc != ATTN_OK) {
      cudaFreeAsync(ws, stream);
      return rc;
    }
    counts = c;
    entries = e;
  }
  p.map_counts = counts;
  p.map_entries = entries;
  const bool sc = softcap > 0.f, al = alibi != nullptr;
  if (fp8) rc = launch_fwd_d<128, true>(dev, tq, tk, tv, p, sc, al, stream);
  else if (pair) rc = launch_pair(dev, tq, tk, tv, p, sc, al, stream);
  else if (D == 128) rc = launch_fwd_d<128, false>(dev, tq, tk, tv, p, sc, al, stream);
  else rc = launch_fwd_d<64, false>(dev, tq, tk, tv, p, sc, al, stream);
  if (ws) cudaFreeAsync(ws, stream);
  return rc;
}

// ---------------------------------------------------------------------------------------
// Allocation-free variant of the document-mask path.
//
// Some callers cannot allocate device memory during a call: code that runs inside a
// framework whose caching allocator owns all of device memory (an outside allocation can
// fail under its memory cap or fragment its pool), serving loops that must not let an
// allocation or free synchronise the device in the middle of a request, and programs that
// reserve a fixed memory budget up front.  For them the tile map that attn_fwd builds in a
// stream-ordered workspace lives instead in the array below, sized for at most
// ATTN_NOALLOC_SCRATCH_BYTES.  Every device that loads this library holds the array until
// the process exits.  The array is shared by all calls on a device: two such calls whose
// kernels overlap on the GPU (different streams, no ordering between them) race on it.
// Nothing in it has to start at zero: each call's map build rewrites every value the
// attention kernel then reads.
// ---------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the array on the current device.  Host code may only use the symbol to
// look this address up (the symbol itself is a host-side stand-in, not a device pointer);
// this is done on the first call on each device, with that device current.
int noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return ATTN_ERR_CUDA;
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return ATTN_OK;
}

int run_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq,
                    int Sk, int D, float scale, int mask_kind, int window, float softcap, const float* alibi,
                    const int* doc_ids, cudaStream_t stream) {
  int rc = check_common(q, k, v, o, lse, B, H, Sq, Sk, D, scale, mask_kind, window, softcap, alibi, doc_ids);
  if (rc != ATTN_OK) return rc;
  const bool need_map = (mask_kind & ATTN_MASK_DOC) != 0;
  if (need_map && B > 65535) return ATTN_ERR_INVALID;   // tile-map grid.y = B
  if (need_map && ws_bytes_for_map(B, Sq, Sk) > static_cast<size_t>(ATTN_NOALLOC_SCRATCH_BYTES))
    return ATTN_ERR_INVALID;   // the tile map would not fit in the fixed array
  int dev = 0;
  if ((rc = current_device(&dev)) != ATTN_OK) return rc;
  void* scratch = nullptr;
  if (need_map && (rc = noalloc_scratch(dev, &scratch)) != ATTN_OK) return rc;

  FwdParams p = make_params(o, lse, B, H, H, Sq, Sk, scale, mask_kind, window, softcap, alibi, doc_ids);
  p.lpt_heads = lpt_head_group(p, Sk, D, 2);
  CUtensorMap tq, tk, tv;
  if (encode_map(&tq, q, false, B * H, Sq, D) != ATTN_OK || encode_map(&tk, k, false, B * H, Sk, D) != ATTN_OK ||
      encode_map(&tv, v, false, B * H, Sk, D) != ATTN_OK)
    return ATTN_ERR_CUDA;
  if (need_map) {
    int* c = static_cast<int*>(scratch);
    uint32_t* e = reinterpret_cast<uint32_t*>(static_cast<char*>(scratch) + ws_counts_bytes(B, Sq));
    int* sorted = reinterpret_cast<int*>(static_cast<char*>(scratch) + ws_counts_bytes(B, Sq) + ws_entries_bytes(B, Sq, Sk));
    if ((rc = launch_tile_map(c, e, B, Sq, Sk, mask_kind, window, doc_ids, stream, sorted)) != ATTN_OK) return rc;
    p.doc_sorted = sorted;
    p.map_counts = c;
    p.map_entries = e;
  }
  const bool sc = softcap > 0.f, al = alibi != nullptr;
  if (D == 128) return launch_fwd_d<128, false>(dev, tq, tk, tv, p, sc, al, stream);
  return launch_fwd_d<64, false>(dev, tq, tk, tv, p, sc, al, stream);
}

// Packed variable-length sequences (token-major tensors).  The work items are
// (sequence, head, 256-row block) up to the longest sequence; blocks past the end of a
// shorter sequence are empty.  The kernel checks each sequence's bounds against the totals
// and the maximum lengths and records ATTN_ERR_INVALID (skipping that sequence) if they fail.
int run_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_q,
                   const int* cu_k, int nseq, int max_sq, int max_sk, int total_q, int total_k, int H, int Hkv,
                   int D, float scale, int mask_kind, int window, float softcap, const float* alibi,
                   cudaStream_t stream) {
  if (!cu_q || !cu_k || nseq <= 0) return ATTN_ERR_INVALID;
  if (total_q <= 0 || total_k <= 0 || max_sq <= 0 || max_sk <= 0) return ATTN_ERR_INVALID;
  if (max_sq > total_q || max_sk > total_k) return ATTN_ERR_INVALID;
  if (mask_kind & ATTN_MASK_DOC) return ATTN_ERR_INVALID;   // sequences already separate documents
  int rc = check_common(q, k, v, o, lse, nseq, H, max_sq, max_sk, D, scale, mask_kind, window, softcap, alibi,
                        nullptr);
  if (rc != ATTN_OK) return rc;
  if (Hkv <= 0 || H % Hkv != 0) return ATTN_ERR_INVALID;
  if (static_cast<long long>(total_q) * H > 0x7fffffffLL || static_cast<long long>(total_k) * Hkv > 0x7fffffffLL)
    return ATTN_ERR_INVALID;
  int dev = 0;
  if ((rc = current_device(&dev)) != ATTN_OK) return rc;
  FwdParams p = make_params(o, lse, nseq, H, Hkv, max_sq, max_sk, scale, mask_kind, window, softcap, alibi, nullptr);
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.Tq = total_q;
  p.Tk = total_k;
  p.lpt_heads = lpt_head_group(p, max_sk, D, 2);
  CUtensorMap tq, tk, tv;
  if (encode_map_thd(&tq, q, H, total_q, D) != ATTN_OK || encode_map_thd(&tk, k, Hkv, total_k, D) != ATTN_OK ||
      encode_map_thd(&tv, v, Hkv, total_k, D) != ATTN_OK)
    return ATTN_ERR_CUDA;
  const bool sc = softcap > 0.f, al = alibi != nullptr;
  if (D == 128) return launch_fwd_d<128, false>(dev, tq, tk, tv, p, sc, al, stream);
  return launch_fwd_d<64, false>(dev, tq, tk, tv, p, sc, al, stream);
}

#include "attn_bwd_api.inc"
#include "attn_fp4_api.inc"

}  // namespace

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq, int Sk,
             int D, float scale, int mask_kind, int window, float softcap, const float* alibi_slopes,
             const int* doc_ids, void* stream) {
  return run_fwd(false, q, k, v, nullptr, nullptr, nullptr, o, lse, B, H, H, Sq, Sk, D, scale, mask_kind, window,
                 softcap, alibi_slopes, doc_ids, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

int attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv,
                 int Sq, int Sk, int D, float scale, int mask_kind, int window, float softcap,
                 const float* alibi_slopes, const int* doc_ids, void* stream) {
  return run_fwd(false, q, k, v, nullptr, nullptr, nullptr, o, lse, B, H, H_kv, Sq, Sk, D, scale, mask_kind,
                 window, softcap, alibi_slopes, doc_ids, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

int attn_fwd_pair(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv,
                  int Sq, int Sk, int D, float scale, int mask_kind, int window, float softcap,
                  const float* alibi_slopes, const int* doc_ids, void* stream) {
  return run_fwd(false, q, k, v, nullptr, nullptr, nullptr, o, lse, B, H, H_kv, Sq, Sk, D, scale, mask_kind,
                 window, softcap, alibi_slopes, doc_ids, nullptr, nullptr, static_cast<cudaStream_t>(stream), true);
}

int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens_q,
                    const int* cu_seqlens_k, int nseq, int max_seqlen_q, int max_seqlen_k, int total_q,
                    int total_k, int H, int H_kv, int D, float scale, int mask_kind, int window, float softcap,
                    const float* alibi_slopes, void* stream) {
  return run_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, nseq, max_seqlen_q, max_seqlen_k, total_q,
                        total_k, H, H_kv, D, scale, mask_kind, window, softcap, alibi_slopes,
                        static_cast<cudaStream_t>(stream));
}

int attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq,
                     int Sk, int D, float scale, int mask_kind, int window, float softcap,
                     const float* alibi_slopes, const int* doc_ids, void* stream) {
  return run_fwd_noalloc(q, k, v, o, lse, B, H, Sq, Sk, D, scale, mask_kind, window, softcap, alibi_slopes,
                         doc_ids, static_cast<cudaStream_t>(stream));
}

int attn_fwd_with_map(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq,
                      int Sk, int D, float scale, int mask_kind, int window, float softcap,
                      const float* alibi_slopes, const int* doc_ids, const int* counts, const uint32_t* entries,
                      void* stream) {
  if (!counts || !entries) return ATTN_ERR_INVALID;
  return run_fwd(false, q, k, v, nullptr, nullptr, nullptr, o, lse, B, H, H, Sq, Sk, D, scale, mask_kind, window,
                 softcap, alibi_slopes, doc_ids, counts, entries, static_cast<cudaStream_t>(stream));
}

int attn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale, const float* k_scale,
                 const float* v_scale, void* o, float* lse, int B, int H, int Sq, int Sk, int D, float scale,
                 int mask_kind, int window, float softcap, const float* alibi_slopes, const int* doc_ids,
                 void* stream) {
  if (!q_scale || !k_scale || !v_scale) return ATTN_ERR_INVALID;
  if (!aligned16(q_scale) || !aligned16(k_scale) || !aligned16(v_scale)) return ATTN_ERR_INVALID;
  return run_fwd(true, q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B, H, H, Sq, Sk, D, scale, mask_kind, window,
                 softcap, alibi_slopes, doc_ids, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
             void* dq, void* dk, void* dv, int B, int H, int H_kv, int Sq, int Sk, int D, float scale,
             int mask_kind, int window, float softcap, const float* alibi_slopes, const int* doc_ids,
             void* stream) {
  return run_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, H_kv, Sq, Sk, D, scale, mask_kind, window, softcap,
                 alibi_slopes, doc_ids, static_cast<cudaStream_t>(stream));
}

int attn_fwd_fp4(const void* q4, const void* k4, const void* vt4, const void* q_sf, const void* k_sf,
                 const void* v_sf, void* o, float* lse, int B, int H, int H_kv, int Sq, int Sk, float scale,
                 void* stream) {
  return run_fwd_fp4(q4, k4, vt4, q_sf, k_sf, v_sf, o, lse, B, H, H_kv, Sq, Sk, scale,
                     static_cast<cudaStream_t>(stream));
}

int attn_quantize_mxfp4(const void* x, void* xq, void* x_sf, int B, int H, int S, int D, int transpose,
                        void* stream) {
  return run_quant_mxfp4(x, xq, x_sf, B, H, S, D, transpose, static_cast<cudaStream_t>(stream));
}

int attn_tile_map_build(int* counts, uint32_t* entries, int B, int Sq, int Sk, int mask_kind, int window,
                        const int* doc_ids, void* stream) {
  if (!counts || !entries) return ATTN_ERR_INVALID;
  if (!aligned16(counts) || !aligned16(entries)) return ATTN_ERR_INVALID;
  if (B <= 0 || Sq <= 0 || Sk <= 0 || Sq > ATTN_MAX_SEQ || Sk > ATTN_MAX_SEQ) return ATTN_ERR_INVALID;
  if (B > 65535) return ATTN_ERR_INVALID;
  if (mask_kind & ~(ATTN_MASK_CAUSAL | ATTN_MASK_WINDOW | ATTN_MASK_DOC)) return ATTN_ERR_INVALID;
  if ((mask_kind & ATTN_MASK_WINDOW) && window <= 0) return ATTN_ERR_INVALID;
  if ((mask_kind & ATTN_MASK_DOC) && (doc_ids == nullptr || Sq != Sk)) return ATTN_ERR_INVALID;
  int dev = 0;
  const int rc = current_device(&dev);
  if (rc != ATTN_OK) return rc;
  return launch_tile_map(counts, entries, B, Sq, Sk, mask_kind, window, doc_ids, static_cast<cudaStream_t>(stream));
}

int attn_quantize_e4m3(const float* x, void* xq, float* scales, int B, int H, int S, int D, void* stream) {
  if (!x || !xq || !scales) return ATTN_ERR_INVALID;
  if (!aligned16(x) || !aligned16(xq) || !aligned16(scales)) return ATTN_ERR_INVALID;
  if (B <= 0 || H <= 0 || S <= 0 || D <= 0 || D % 16 != 0 || D > 256 || S > ATTN_MAX_SEQ) return ATTN_ERR_INVALID;
  int dev = 0;
  const int rc = current_device(&dev);
  if (rc != ATTN_OK) return rc;
  const int nsb = (S + 127) / 128;
  const long long grid = static_cast<long long>(B) * H * nsb;
  if (grid > 0x7fffffffLL) return ATTN_ERR_INVALID;
  if (D <= 128)
    attn::quant_e4m3_kernel<8><<<static_cast<unsigned>(grid), attn::kQuantThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        x, static_cast<uint8_t*>(xq), scales, S, D, nsb);
  else
    attn::quant_e4m3_kernel<16><<<static_cast<unsigned>(grid), attn::kQuantThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        x, static_cast<uint8_t*>(xq), scales, S, D, nsb);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_get_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, attn::g_attn_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(attn::g_attn_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  return v;
}

const char* attn_strerror(int code) {
  switch (code) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported device (needs compute capability 10.0, B200)";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    case ATTN_ERR_NOMEM: return "workspace allocation failed";
    case ATTN_ERR_CHECK: return "a bounds check of the debug build failed inside a kernel";
    default: return "unknown status";
  }
}

void attn_shutdown(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  cudaMemPool_t pool;
  if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) cudaMemPoolTrimTo(pool, 0);
}

#ifdef ATTN_ABLATION
int attn_ablation_set(float tau) {
  if (!std::isfinite(tau) || tau < 0.f || tau > 8.f) return ATTN_ERR_INVALID;   // P <= 2^tau <= 256
  int dev = 0;
  const int rc = current_device(&dev);
  if (rc != ATTN_OK) return rc;
  const unsigned long long zero[2] = {0ull, 0ull};
  if (cudaMemcpyToSymbol(attn::g_abl_tau, &tau, sizeof(float)) != cudaSuccess ||
      cudaMemcpyToSymbol(attn::g_abl_counts, zero, sizeof(zero)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return ATTN_OK;
}

int attn_ablation_counts(unsigned long long* out) {
  if (!out) return ATTN_ERR_INVALID;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpyFromSymbol(out, attn::g_abl_counts, 2 * sizeof(unsigned long long)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return ATTN_OK;
}

int attn_ablation_sw_exp_every(void) { return attn::kSwExpEvery; }
#endif

void attn_debug_set_fault(int skip_signal, int timeout_ms) {
  g_fault_skip.store(skip_signal ? 1 : 0);
  g_timeout_ms.store(timeout_ms > 0 ? timeout_ms : 1000);
}

}  // extern "C"
