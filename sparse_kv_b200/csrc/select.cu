// select.cu -- centroid scoring and top-k cluster choice
// ("Squeezed Attention" Q2 step 2: compare the query with every cluster
// centroid and keep the most similar clusters; their keys are attended next).
//
// One CTA per KV group (b, kvh).  The group's query heads are summed once
// (one selection per GQA group, the cheapest form of the query-centroid
// comparison).  Centroid rows stream into shared memory in 64 KiB chunks by
// bulk-async copies (two stages), each row is scored by 16 lanes with 16-byte
// shared loads and a shuffle reduction.  A radix select over order-preserving
// 32-bit score keys finds the k-th largest score; the kept clusters are those
// above it plus the lowest-index ones equal to it (ties to the lower index),
// written in ascending id order with their key ranges.
#include "common.cuh"
#include "decode.cuh"

namespace skv {
namespace {

constexpr int kSelThreads = 512;
constexpr int kMaxClusters = 4096;
constexpr int kChunk = 256;                             // centroids per stage
constexpr int kChunkBytes = kChunk * kHeadDim * 2;      // 64 KiB
constexpr int kSelStages = 2;
// shared memory: stages | keys u32[kMaxClusters] | q sum f32[128] | flags u8[kMaxClusters] |
//                histogram int[256] | warp sums int[16] | scalars int[4] | mbarriers
constexpr size_t kOffKeys = (size_t)kSelStages * kChunkBytes;
constexpr size_t kOffQ = kOffKeys + sizeof(uint32_t) * kMaxClusters;
constexpr size_t kOffFlag = kOffQ + 128 * 4;
constexpr size_t kOffHist = kOffFlag + kMaxClusters;
constexpr size_t kOffWsum = kOffHist + 256 * 4;
constexpr size_t kOffScal = kOffWsum + 16 * 4;
constexpr size_t kOffBar = kOffScal + 16;
constexpr size_t kSelSmem = kOffBar + kSelStages * 8;

// Order-preserving map of an fp32 score to an unsigned key.
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix of per-thread counts (threads own contiguous
// runs in index order); returns the thread's offset, total in *total.
__device__ __forceinline__ int block_exclusive_scan(int cnt, int* wsum, int* total) {
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
  for (int w = 0; w < kSelThreads / 32; ++w) {
    if (w < warp) base += wsum[w];
    tot += wsum[w];
  }
  __syncthreads();
  *total = tot;
  return base + incl - cnt;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(const uint16_t* __restrict__ q,
                                                            const uint16_t* __restrict__ cent,
                                                            const int* __restrict__ off, int Hq,
                                                            int Hkv, int C, int k, int* ids, int* ss,
                                                            int* se) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t* key = reinterpret_cast<uint32_t*>(smem + kOffKeys);
  float* qs = reinterpret_cast<float*>(smem + kOffQ);
  unsigned char* flag = smem + kOffFlag;
  int* hist = reinterpret_cast<int*>(smem + kOffHist);
  int* wsum = reinterpret_cast<int*>(smem + kOffWsum);
  int* scal = reinterpret_cast<int*>(smem + kOffScal);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);

  const int g = blockIdx.x, b = g / Hkv, kvh = g % Hkv, G = Hq / Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nchunks = (C + kChunk - 1) / kChunk;
  const unsigned char* cg = reinterpret_cast<const unsigned char*>(cent + (size_t)g * C * kHeadDim);

  // Centroid rows stream through kSelStages shared-memory stages by bulk copy.
  auto issue = [&](int chunk) {
    const int st = chunk % kSelStages;
    const int rows = min(kChunk, C - chunk * kChunk);
    const uint32_t bytes = (uint32_t)rows * kHeadDim * 2;
    mbar_arrive_expect_tx(&bar[st], bytes);
    const unsigned char* src = cg + (size_t)chunk * kChunkBytes;
    unsigned char* dst = smem + (size_t)st * kChunkBytes;
    for (uint32_t o = 0; o < bytes; o += 16384)
      bulk_load(dst + o, src + o, min(16384u, bytes - o), &bar[st], policy_evict_first());
  };
  if (tid == 0) {
    for (int i = 0; i < kSelStages; ++i) mbar_init(&bar[i], 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0)
    for (int i = 0; i < kSelStages && i < nchunks; ++i) issue(i);

  if (tid < kHeadDim) {
    float sum = 0.f;
    for (int h = 0; h < G; ++h)
      sum += __uint_as_float((uint32_t)q[((size_t)b * Hq + kvh * G + h) * kHeadDim + tid] << 16);
    qs[tid] = sum;
  }
  for (int c = tid; c < C; c += kSelThreads) flag[c] = 0;
  __syncthreads();

  // ---- scores: 16 lanes per centroid row (8 dims each), 2 rows per warp step
  const int ch = lane & 15;
  float qv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qv[e] = qs[ch * 8 + e];
  for (int chunk = 0; chunk < nchunks; ++chunk) {
    const int st = chunk % kSelStages;
    if (!mbar_wait_bounded(&bar[st], (chunk / kSelStages) & 1, nullptr)) break;
    const unsigned char* sc = smem + (size_t)st * kChunkBytes;
    const int rows = min(kChunk, C - chunk * kChunk);
#pragma unroll 4
    for (int rb = warp * 2; rb < rows; rb += (kSelThreads / 32) * 2) {  // warp-uniform bound
      const int r = rb + (lane >> 4);
      const bool valid = r < rows;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (valid) w = *reinterpret_cast<const uint4*>(sc + (size_t)r * kHeadDim * 2 + ch * 16);
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
      if (valid && ch == 0) key[chunk * kChunk + r] = score_key(acc);
    }
    __syncthreads();  // stage st fully read
    if (tid == 0 && chunk + kSelStages < nchunks) issue(chunk + kSelStages);
  }
  __syncthreads();

  // ---- radix select: the k-th largest key T, 8 bits at a time from the top
  uint32_t prefix = 0, pmask = 0;
  int kk = k;  // rank still to find below the fixed prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int c = tid; c < C; c += kSelThreads) {
      const uint32_t kc = key[c];
      if ((kc & pmask) == prefix) atomicAdd(&hist[(kc >> shift) & 0xFFu], 1);
    }
    __syncthreads();
    if (warp == 0) {  // bins from the top: find the digit holding rank kk
      int cnt[8], run = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = hist[255 - (lane * 8 + j)];
        run += cnt[j];
      }
      int incl = run;  // inclusive prefix over lanes (bins in descending order)
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, m);
        if (lane >= m) incl += y;
      }
      int before = incl - run;
      const bool mine = before < kk && kk <= incl;
      if (mine) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (before < kk && kk <= before + cnt[j]) {
            scal[0] = 255 - (lane * 8 + j);  // digit
            scal[1] = kk - before;           // rank within that digit
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
  const uint32_t T = prefix;  // the k-th largest key; kk of the keys equal to T are taken

  // ---- flags: keys above T, plus the first kk keys equal to T in index order
  const int per = (C + kSelThreads - 1) / kSelThreads;
  const int c0 = tid * per;
  int nties = 0;
  for (int c = c0; c < c0 + per && c < C; ++c) nties += (key[c] == T);
  int tot = 0;
  int tie_rank = block_exclusive_scan(nties, wsum, &tot);
  int cnt = 0;
  for (int c = c0; c < c0 + per && c < C; ++c) {
    const uint32_t kc = key[c];
    int f = kc > T;
    if (kc == T) f = (tie_rank++ < kk);
    flag[c] = (unsigned char)f;
    cnt += f;
  }

  // ---- compact in ascending id order
  int pos = block_exclusive_scan(cnt, wsum, &tot);
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
  const size_t smem = kSelSmem;
  static std::atomic<bool> attr_set[64];  // per device; racing first calls only repeat the set-up
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return (int)e;
    attr_set[dev] = true;
  }
  select_kernel<<<B * Hkv, kSelThreads, smem, static_cast<cudaStream_t>(stream)>>>(
      q, cent, off, Hq, Hkv, C, k, ids, ss, se);
  return (int)cudaGetLastError();
}

}  // namespace skv
