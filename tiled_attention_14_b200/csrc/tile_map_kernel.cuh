// tile_map_kernel.cuh — block-sparse tile map builder (EMPTY / PARTIAL / FULL per
// (256-row query block, 128-column key tile), exact).
//
// FlexAttention skips blocks that its mask removes entirely (page "PyTorch's
// FlexAttention mit FlashAttention-4 ist ein Game-Changer", section "Aktuelle
// Einschränkungen", block sparsity).  This kernel builds the list of key tiles each query
// block must visit, with one class per 128-row query tile, in the C-ABI's entry format
// (kt | class0 << 24 | class1 << 26).
//
// One CTA per (query block, b), one thread per query row.  Each row's visible keys under
// the causal / window bits form one interval [jlo, jhi].  With document masking:
//  * if doc_ids[b, :] is non-decreasing (the running document index), each document is
//    one run, so the row's document is the interval found by two binary searches and the
//    visible set stays one interval: every (row, tile) test is O(1);
//  * otherwise the kernel tests every (row, key) pair of the tile (exact, slower).
// Per tile the rows' answers are reduced per query tile with warp votes and shared memory,
// then the non-empty tiles are compacted in increasing order with a block prefix sum.
// Optionally it records, per batch row, whether the document ids are non-decreasing (the
// attention kernel then tests documents as key intervals instead of element by element).
#pragma once
#include <cstdint>

namespace attn {

constexpr int kMapThreads = 256;
constexpr int kMapChunk = 256;   // key tiles classified per pass

__device__ __forceinline__ int lower_bound_i32(const int* a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(a + mid) < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}
__device__ __forceinline__ int upper_bound_i32(const int* a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(a + mid) <= v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kMapThreads)
tile_map_kernel(int* __restrict__ counts, uint32_t* __restrict__ entries, int Sq, int Sk,
                int mask_kind, int window, const int* __restrict__ doc, int nqb, int nkt,
                int* __restrict__ sorted_flags) {
  __shared__ uint8_t w_any[8][kMapChunk];
  __shared__ uint8_t w_all[8][kMapChunk];
  __shared__ int kdoc[128];
  __shared__ int warp_cnt[8];
  __shared__ int running;

  const int qb = blockIdx.x, b = blockIdx.y;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int row = qb * 256 + t;
  const bool valid = row < Sq;
  const int ip = row + (Sk - Sq);
  const bool causal = mask_kind & 1, win = mask_kind & 2, has_doc = mask_kind & 4;

  int jlo = win ? ip - window + 1 : 0;
  int jhi = causal ? ip : (win ? ip + window - 1 : Sk - 1);
  jlo = max(jlo, 0);
  jhi = min(jhi, Sk - 1);

  const int* drow = has_doc ? doc + static_cast<size_t>(b) * Sk : nullptr;
  bool sorted = true;
  int mydoc = 0;
  if (has_doc) {
    for (int j = t; j + 1 < Sk; j += kMapThreads)
      if (__ldg(drow + j) > __ldg(drow + j + 1)) sorted = false;
    sorted = __syncthreads_and(sorted);
    if (sorted_flags != nullptr && qb == 0 && t == 0) sorted_flags[b] = sorted ? 1 : 0;
    if (valid) {
      mydoc = __ldg(drow + row);
      if (sorted) {
        jlo = max(jlo, lower_bound_i32(drow, Sk, mydoc));
        jhi = min(jhi, upper_bound_i32(drow, Sk, mydoc) - 1);
      }
    }
  }
  if (t == 0) running = 0;
  __syncthreads();

  uint32_t* out = entries + (static_cast<size_t>(b) * nqb + qb) * nkt;
  for (int chunk = 0; chunk < nkt; chunk += kMapChunk) {
    const int nk = min(kMapChunk, nkt - chunk);
    for (int k = 0; k < nk; ++k) {
      const int kt = chunk + k;
      const int c0 = kt * 128, c1 = c0 + 127, c1v = min(c1, Sk - 1);
      bool any, all;
      if (!has_doc || sorted) {
        any = valid && jlo <= jhi && jlo <= c1v && jhi >= c0;
        all = !valid || (c1 <= Sk - 1 && jlo <= c0 && jhi >= c1);
      } else {
        __syncthreads();
        if (t < 128) kdoc[t] = (c0 + t < Sk) ? __ldg(drow + c0 + t) : 0;
        __syncthreads();
        int cnt = 0;
        if (valid) {
          for (int c = 0; c < 128; ++c) {
            const int j = c0 + c;
            cnt += (j <= c1v && j >= jlo && j <= jhi && kdoc[c] == mydoc) ? 1 : 0;
          }
        }
        any = valid && cnt > 0;
        all = !valid || (cnt == 128);
      }
      const bool wa = __any_sync(0xffffffffu, any);
      const bool wl = __all_sync(0xffffffffu, all);
      if (lane == 0) {
        w_any[warp][k] = wa;
        w_all[warp][k] = wl;
      }
    }
    __syncthreads();
    // thread k combines the four warps of each query tile for key tile chunk + k
    uint32_t entry = 0;
    bool keep = false;
    if (t < nk) {
      int cls[2];
      for (int g = 0; g < 2; ++g) {
        bool a = false, l = true;
        for (int w = 4 * g; w < 4 * g + 4; ++w) {
          a = a || w_any[w][t];
          l = l && w_all[w][t];
        }
        cls[g] = !a ? 0 : (l ? 2 : 1);
      }
      keep = cls[0] != 0 || cls[1] != 0;
      entry = static_cast<uint32_t>(chunk + t) | (static_cast<uint32_t>(cls[0]) << 24) |
              (static_cast<uint32_t>(cls[1]) << 26);
    }
    // block exclusive prefix sum of `keep`
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int off = running;
    for (int w = 0; w < warp; ++w) off += warp_cnt[w];
    off += __popc(bal & ((1u << lane) - 1u));
    if (keep) out[off] = entry;
    __syncthreads();
    if (t == 0) {
      int tot = 0;
      for (int w = 0; w < 8; ++w) tot += warp_cnt[w];
      running += tot;
    }
    __syncthreads();
  }
  if (t == 0) counts[b * nqb + qb] = running;
}

}  // namespace attn
