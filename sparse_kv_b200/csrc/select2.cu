// select2.cu -- two-level centroid selection ("Squeezed Attention" Q2 step 4:
// hierarchical clustering of the fixed context; at lookup the query first
// picks the most relevant coarse clusters, then only the fine clusters inside
// them are compared, so far fewer centroids are read than in a flat search).
//
// One CTA per KV group (b, kvh), with the group's query heads summed once (as
// the one-level selection does):
//   1. score the C1 coarse centroids, keep the k1 best (ties to the lower id);
//   2. the fine clusters of the kept coarse clusters (coarse cluster i owns
//      fine clusters coarse_off[i] .. coarse_off[i+1]-1) are the candidates,
//      listed in ascending id order;
//   3. score the candidates' fine centroids only, keep the min(k2, #candidates)
//      best (ties to the lower id) and write their ids ascending with their key
//      ranges; unused output slots get id -1 and an empty range.
// Both top-k steps are a radix select over order-preserving 32-bit score keys
// in shared memory.  Centroid rows are read straight from global memory with
// 16-byte loads (16 lanes per row): at these sizes (a few hundred rows per
// group) the loads of all rows of a pass are in flight at once.
#include <cuda_runtime.h>

#include "../../include/sparsekv.h"
#include "common.cuh"

namespace skv {
namespace {

constexpr int kS2Threads = 512;
constexpr int kS2MaxCoarse = 1024;
constexpr int kS2MaxFine = 4096;

__device__ __forceinline__ uint32_t s2_key(float s) {  // order-preserving fp32 -> u32
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix over the block of per-thread counts (threads own runs in
// index order); the total in *total.
__device__ __forceinline__ int s2_scan(int cnt, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = cnt;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, m);
    if (lane >= m) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int base = 0, tot = 0;
  for (int w = 0; w < kS2Threads / 32; ++w) {
    if (w < warp) base += wsum[w];
    tot += wsum[w];
  }
  __syncthreads();
  *total = tot;
  return base + incl - cnt;
}

// Score rows: key[j] = score_key(qs . row(j)), 16 lanes per row.
template <typename RowPtr>
__device__ __forceinline__ void s2_score(const float* qs, int n, RowPtr row, uint32_t* key) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, ch = lane & 15;
  float qv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qv[e] = qs[ch * 8 + e];
  for (int rb = warp * 2; rb < n; rb += (kS2Threads / 32) * 2) {  // warp-uniform bound
    const int r = rb + (lane >> 4);
    const bool valid = r < n;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (valid) w = __ldg(reinterpret_cast<const uint4*>(row(r) + ch * 8));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      acc = fmaf(qv[2 * u], __uint_as_float(ws[u] << 16), acc);
      acc = fmaf(qv[2 * u + 1], __uint_as_float(ws[u] & 0xFFFF0000u), acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 8);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (valid && ch == 0) key[r] = s2_key(acc);
  }
  __syncthreads();
}

// Top-k of key[0..n) (1 <= k <= n): flag[j] = 1 for the k largest keys, ties
// to the lower index.  Radix select, 8 bits at a time from the top.
__device__ void s2_topk(const uint32_t* key, int n, int k, unsigned char* flag, int* hist, int* wsum,
                        int* scal) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, pmask = 0;
  int kk = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kS2Threads) hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += kS2Threads) {
      const uint32_t kj = key[j];
      if ((kj & pmask) == prefix) atomicAdd(&hist[(kj >> shift) & 0xFFu], 1);
    }
    __syncthreads();
    if (warp == 0) {
      int cnt[8], run = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = hist[255 - (lane * 8 + j)];
        run += cnt[j];
      }
      int incl = run;
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, m);
        if (lane >= m) incl += y;
      }
      int before = incl - run;
      if (before < kk && kk <= incl) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (before < kk && kk <= before + cnt[j]) {
            scal[0] = 255 - (lane * 8 + j);
            scal[1] = kk - before;
          }
          before += cnt[j];
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)scal[0] << shift;
    pmask |= 0xFFu << shift;
    kk = scal[1];
    __syncthreads();
  }
  const uint32_t T = prefix;  // the k-th largest key; kk of the keys equal to T are kept
  const int per = (n + kS2Threads - 1) / kS2Threads;
  const int j0 = tid * per;
  int nties = 0;
  for (int j = j0; j < j0 + per && j < n; ++j) nties += (key[j] == T);
  int tot = 0;
  int tie_rank = s2_scan(nties, wsum, &tot);
  for (int j = j0; j < j0 + per && j < n; ++j) {
    const uint32_t kj = key[j];
    int f = kj > T;
    if (kj == T) f = (tie_rank++ < kk);
    flag[j] = (unsigned char)f;
  }
  __syncthreads();
}

struct S2Smem {
  float qs[128];
  uint32_t key[kS2MaxFine];
  int cand[kS2MaxFine];
  unsigned char flag[kS2MaxFine];
  int hist[256];
  int wsum[kS2Threads / 32];
  int scal[4];
};

__global__ void __launch_bounds__(kS2Threads) select2_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ coarse, const int* __restrict__ coarse_off,
    const uint16_t* __restrict__ fine, const int* __restrict__ cluster_off, int Hq, int Hkv, int C1, int C,
    int k1, int k2, int* ids, int* ss, int* se) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  S2Smem& S = *reinterpret_cast<S2Smem*>(smem_raw);
  const int g = blockIdx.x, b = g / Hkv, kvh = g % Hkv, G = Hq / Hkv;
  const int tid = threadIdx.x;
  if (tid < kHeadDim) {
    float sum = 0.f;
    for (int h = 0; h < G; ++h)
      sum += __uint_as_float((uint32_t)q[((size_t)b * Hq + kvh * G + h) * kHeadDim + tid] << 16);
    S.qs[tid] = sum;
  }
  __syncthreads();

  // ---- level 1: the k1 best coarse clusters
  const uint16_t* cg = coarse + (size_t)g * C1 * kHeadDim;
  s2_score(S.qs, C1, [&](int r) { return cg + (size_t)r * kHeadDim; }, S.key);
  s2_topk(S.key, C1, k1, S.flag, S.hist, S.wsum, S.scal);

  // ---- candidates: the fine clusters of the kept coarse clusters, ascending
  // (ranges clamped to [0, C) and the list to kS2MaxFine: a malformed
  // coarse_off cannot write outside the shared arrays)
  const int* og1 = coarse_off + (size_t)g * (C1 + 1);
  auto lo = [&](int c) { return min(max(og1[c], 0), C); };
  auto hi = [&](int c) { return max(min(og1[c + 1], C), lo(c)); };
  const int per1 = (C1 + kS2Threads - 1) / kS2Threads;
  const int c0 = tid * per1;
  int mine = 0;
  for (int c = c0; c < c0 + per1 && c < C1; ++c)
    if (S.flag[c]) mine += hi(c) - lo(c);
  int n_cand = 0;
  int pos = s2_scan(mine, S.wsum, &n_cand);
  for (int c = c0; c < c0 + per1 && c < C1; ++c)
    if (S.flag[c])
      for (int f = lo(c); f < hi(c); ++f) {
        if (pos < kS2MaxFine) S.cand[pos] = f;
        ++pos;
      }
  n_cand = min(n_cand, kS2MaxFine);
  __syncthreads();

  // ---- level 2: the best candidates
  const uint16_t* fg = fine + (size_t)g * C * kHeadDim;
  const int kk = min(k2, n_cand);
  if (kk > 0) {
    s2_score(S.qs, n_cand, [&](int r) { return fg + (size_t)S.cand[r] * kHeadDim; }, S.key);
    s2_topk(S.key, n_cand, kk, S.flag, S.hist, S.wsum, S.scal);
  }

  // ---- compact in ascending id order, then the unused slots
  const int per2 = (n_cand + kS2Threads - 1) / kS2Threads;
  const int j0 = tid * per2;
  int cnt = 0;
  if (kk > 0)
    for (int j = j0; j < j0 + per2 && j < n_cand; ++j) cnt += S.flag[j];
  int tot = 0;
  int at = s2_scan(cnt, S.wsum, &tot);
  const size_t ob = (size_t)g * k2;
  const int* og = cluster_off + (size_t)g * (C + 1);
  if (kk > 0)
    for (int j = j0; j < j0 + per2 && j < n_cand; ++j)
      if (S.flag[j]) {
        const int f = S.cand[j];
        ids[ob + at] = f;
        ss[ob + at] = og[f];
        se[ob + at] = og[f + 1];
        ++at;
      }
  for (int i = kk + tid; i < k2; i += kS2Threads) {
    ids[ob + i] = -1;
    ss[ob + i] = 0;
    se[ob + i] = 0;
  }
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace skv

extern "C" {

SKV_API skv_status attn_select_centroids2(const void* q, const void* coarse, const int32_t* coarse_off,
                                          const void* fine, const int32_t* cluster_off, int batch,
                                          int q_heads, int kv_heads, int head_dim, int n_coarse,
                                          int n_fine, int k1, int k2, int32_t* sel_ids,
                                          int32_t* seg_start, int32_t* seg_end, skv_stream_t stream) {
  using namespace skv;
  if (!q || !coarse || !coarse_off || !fine || !cluster_off || !sel_ids || !seg_start || !seg_end)
    return SKV_EINVAL;
  if (batch < 1 || q_heads < 1 || kv_heads < 1 || q_heads % kv_heads != 0) return SKV_EINVAL;
  if (head_dim != kHeadDim) return SKV_EUNSUPPORTED;
  if (n_coarse < 1 || n_fine < 1 || k1 < 1 || k1 > n_coarse || k2 < 1 || k2 > n_fine) return SKV_EINVAL;
  if (n_coarse > kS2MaxCoarse || n_fine > kS2MaxFine) return SKV_EUNSUPPORTED;
  if (!aligned16(coarse) || !aligned16(fine)) return SKV_EINVAL;
  const size_t smem = sizeof(S2Smem);
  static std::atomic<bool> attr_set[64];  // per device; racing first calls only repeat the set-up
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SKV_ECUDA;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(select2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return SKV_ECUDA;
    attr_set[dev] = true;
  }
  select2_kernel<<<batch * kv_heads, kS2Threads, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(coarse), coarse_off,
      static_cast<const uint16_t*>(fine), cluster_off, q_heads, kv_heads, n_coarse, n_fine, k1, k2,
      sel_ids, seg_start, seg_end);
  return cudaGetLastError() == cudaSuccess ? SKV_OK : SKV_ECUDA;
}

}  // extern "C"
