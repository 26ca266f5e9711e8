// select.cu -- centroid scoring and top-k cluster choice
// ("Squeezed Attention" Q2 step 2: compare the query with every cluster
// centroid and keep the most similar clusters; their keys are attended next).
//
// One CTA per KV group (b, kvh).  The group's query heads are summed once
// (one selection per GQA group, the cheapest form of the query-centroid
// comparison), each centroid row is scored by 16 lanes with 16-byte loads and
// a shuffle reduction, then a shared-memory bitonic sort over
// (score, -index) keys gives the top k (ties to the lower index), which are
// written in ascending id order with their key ranges.
#include "common.cuh"
#include "decode.cuh"

namespace skv {
namespace {

constexpr int kSelThreads = 512;
constexpr int kMaxClusters = 4096;

__device__ __forceinline__ uint64_t make_key(float s, int c) {
  uint32_t u = __float_as_uint(s);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // order-preserving map
  return ((uint64_t)u << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)c);
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(const uint16_t* __restrict__ q,
                                                            const uint16_t* __restrict__ cent,
                                                            const int* __restrict__ off, int Hq,
                                                            int Hkv, int C, int k, int* ids, int* ss,
                                                            int* se) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint64_t* key = reinterpret_cast<uint64_t*>(smem);                              // [Cp]
  float* qs = reinterpret_cast<float*>(smem + sizeof(uint64_t) * kMaxClusters);   // [128]
  unsigned char* flag = smem + sizeof(uint64_t) * kMaxClusters + 128 * 4;          // [C]
  int* wsum = reinterpret_cast<int*>(flag + kMaxClusters);                        // [16]

  const int g = blockIdx.x, b = g / Hkv, kvh = g % Hkv, G = Hq / Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int Cp = 1;
  while (Cp < C) Cp <<= 1;

  if (tid < kHeadDim) {
    float s = 0.f;
    for (int h = 0; h < G; ++h)
      s += __uint_as_float((uint32_t)q[((size_t)b * Hq + kvh * G + h) * kHeadDim + tid] << 16);
    qs[tid] = s;
  }
  for (int c = tid; c < Cp; c += kSelThreads) key[c] = 0ull;  // padding sorts last
  for (int c = tid; c < C; c += kSelThreads) flag[c] = 0;
  __syncthreads();

  // ---- scores: 16 lanes per centroid row, 2 rows per warp step
  const int ch = lane & 15;
  float qv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qv[e] = qs[ch * 8 + e];
  const uint16_t* cg = cent + (size_t)g * C * kHeadDim;
  const int nw = kSelThreads / 32;
#pragma unroll 4
  for (int cb = warp * 2; cb < C; cb += nw * 2) {  // warp-uniform trip count
    const int c = cb + (lane >> 4);
    const bool valid = c < C;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (valid) w = *reinterpret_cast<const uint4*>(cg + (size_t)c * kHeadDim + ch * 8);
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
    if (valid && ch == 0) key[c] = make_key(acc, c);
  }
  __syncthreads();

  // ---- bitonic sort, descending
  for (int size = 2; size <= Cp; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = tid; t < Cp / 2; t += kSelThreads) {
        const int i = 2 * t - (t & (stride - 1));
        const int j = i + stride;
        const bool desc = (i & size) == 0;
        const uint64_t a = key[i], bb = key[j];
        if ((a < bb) == desc) {
          key[i] = bb;
          key[j] = a;
        }
      }
      __syncthreads();
    }
  }
  for (int r = tid; r < k; r += kSelThreads)
    flag[0xFFFFFFFFu - (uint32_t)(key[r] & 0xFFFFFFFFull)] = 1;
  __syncthreads();

  // ---- compact the flags in ascending id order (each thread owns a run of ids)
  const int per = (C + kSelThreads - 1) / kSelThreads;
  const int c0 = tid * per;
  int cnt = 0;
  for (int c = c0; c < c0 + per && c < C; ++c) cnt += flag[c];
  int incl = cnt;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, m);
    if (lane >= m) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += wsum[w];
  int pos = base + incl - cnt;
  const size_t ob = (size_t)g * k;
  const int* og = off + (size_t)g * (C + 1);
  for (int c = c0; c < c0 + per && c < C; ++c) {
    if (flag[c]) {
      ids[ob + pos] = c;
      ss[ob + pos] = og[c];
      se[ob + pos] = og[c + 1];
      ++pos;
    }
  }
}

}  // namespace

int launch_select(const uint16_t* q, const uint16_t* cent, const int* off, int B, int Hq, int Hkv,
                  int C, int k, int* ids, int* ss, int* se, void* stream) {
  const size_t smem = sizeof(uint64_t) * kMaxClusters + 128 * 4 + kMaxClusters + 16 * 4;
  cudaError_t e =
      cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  select_kernel<<<B * Hkv, kSelThreads, smem, static_cast<cudaStream_t>(stream)>>>(
      q, cent, off, Hq, Hkv, C, k, ids, ss, se);
  return (int)cudaGetLastError();
}

}  // namespace skv
