// select.cu -- centroid scoring and top-k cluster choice
// ("Squeezed Attention" Q2 step 2: compare the query with every cluster
// centroid and keep the most similar clusters; their keys are attended next).
//
// The query heads of a GQA group are summed once (one selection per KV
// group), and score_c = qsum . centroid_c.  The kept clusters are the k best
// scores, ties to the lower index, written in ascending id order with their
// key ranges.  Per-sequence centroids (attn_select_centroids): a CTA pair
// (cluster of 2) per KV group, each CTA bulk-copying and scoring half of the
// group's centroid rows (an SM's copy throughput, not DRAM, bounds the
// scoring at one CTA per group) and storing the keys into the first CTA's
// shared memory, which then selects.
//
// Shared centroids (attn_select_centroids_shared): a thread-block cluster of S
// CTAs shares the centroid rows of one KV head: CTA r bulk-copies rows
// [r C / S, (r + 1) C / S) into a shared-memory ring (no multicast) and scores
// them against every query it serves.  Each
// score goes, as an order-preserving 32-bit key, straight into the shared
// memory of the CTA that owns that query's selection (st.shared::cluster);
// after its last row the CTA arrives remotely on every owner's gather barrier.
// An owner then finds the k-th largest key by a radix select (8 bits per pass,
// warp-aggregated histogram updates, early exit once the boundary digit holds
// exactly the keys still needed) and writes the kept ids in ascending order.
// One cluster per KV head and up to 8 requests ("Squeezed Attention" Q1: one
// fixed context clustered once, reused by every request): CTA j owns request
// j's selection, and every centroid row is read once for all of the cluster's
// requests.
#include "common.cuh"
#include "decode.cuh"

namespace skv {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kMaxClusters = 4096;
constexpr int kSelMaxQ = 8;                         // queries scored per CTA
constexpr int kStageRows = 128;                     // centroid rows per ring stage
constexpr int kStageBytes = kStageRows * kRowBytes;  // 32 KiB
constexpr int kSelStages = 2;
// shared memory: ring | keys u32[kMaxClusters] | query sums f32[kSelMaxQ][128] |
//                histogram int[256] | warp sums int[16] | scalars int[4] | mbarriers
constexpr size_t kOffKeys = (size_t)kSelStages * kStageBytes;
constexpr size_t kOffQ = kOffKeys + sizeof(uint32_t) * kMaxClusters;
constexpr size_t kOffHist = kOffQ + (size_t)kSelMaxQ * kHeadDim * 4;
constexpr size_t kOffWsum = kOffHist + 256 * 4;
constexpr size_t kOffScal = kOffWsum + kSelWarps * 4;
constexpr size_t kOffBar = kOffScal + 16;
constexpr size_t kSelSmem = kOffBar + (kSelStages + 1) * 8;
static_assert(kOffKeys % 16 == 0 && kOffQ % 16 == 0 && kOffBar % 8 == 0, "alignment");

// Per-sequence centroids (attn_select_centroids): one CTA per KV group (b, kvh),
// the group's query heads summed once.  Centroid rows stream into shared
// memory in 64 KiB chunks by bulk-async copies (two stages); each row is scored
// by 16 lanes with 16-byte shared loads and a shuffle reduction.  A radix
// select over order-preserving 32-bit score keys finds the k-th largest score;
// the kept clusters are those above it plus the lowest-index ones equal to it,
// written in ascending id order with their key ranges.  (Splitting a group's
// centroids over a cluster of CTAs, as the shared-centroid kernel below does for
// its requests, measured slower here: the radix select on one CTA per group is
// the critical path, and the cluster's set-up and gather only add to it.)
constexpr int kSeqThreads = 512;
constexpr int kSeqMaxClusters = 4096;
constexpr int kSeqChunk = 256;                             // centroids per stage
constexpr int kSeqChunkBytes = kSeqChunk * kHeadDim * 2;      // 64 KiB
constexpr int kSeqStages = 2;
// shared memory: stages | keys u32[kSeqMaxClusters] | q sum f32[128] | flags u8[kSeqMaxClusters] |
//                histogram int[256] | warp sums int[16] | scalars int[4] | mbarriers
constexpr size_t kSeqOffKeys = (size_t)kSeqStages * kSeqChunkBytes;
constexpr size_t kSeqOffQ = kSeqOffKeys + sizeof(uint32_t) * kSeqMaxClusters;
constexpr size_t kSeqOffFlag = kSeqOffQ + 128 * 4;
constexpr size_t kSeqOffHist = kSeqOffFlag + kSeqMaxClusters;
constexpr size_t kSeqOffWsum = kSeqOffHist + 256 * 4;
constexpr size_t kSeqOffScal = kSeqOffWsum + 16 * 4;
constexpr size_t kSeqOffBar = kSeqOffScal + 16;
constexpr size_t kSeqSmem = kSeqOffBar + kSeqStages * 8;

// ---- thread-block cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Order-preserving map of an fp32 score to an unsigned key.
__device__ __forceinline__ uint32_t seq_score_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix of per-thread counts (threads own contiguous
// runs in index order); returns the thread's offset, total in *total.
__device__ __forceinline__ int seq_block_scan(int cnt, int* wsum, int* total) {
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
  for (int w = 0; w < kSeqThreads / 32; ++w) {
    if (w < warp) base += wsum[w];
    tot += wsum[w];
  }
  __syncthreads();
  *total = tot;
  return base + incl - cnt;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kSeqThreads) select_seq_kernel(const uint16_t* __restrict__ q,
                                                            const uint16_t* __restrict__ cent,
                                                            const int* __restrict__ off, int Hq,
                                                            int Hkv, int C, int k, int* ids, int* ss,
                                                            int* se) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t* key = reinterpret_cast<uint32_t*>(smem + kSeqOffKeys);
  float* qs = reinterpret_cast<float*>(smem + kSeqOffQ);
  unsigned char* flag = smem + kSeqOffFlag;
  int* hist = reinterpret_cast<int*>(smem + kSeqOffHist);
  int* wsum = reinterpret_cast<int*>(smem + kSeqOffWsum);
  int* scal = reinterpret_cast<int*>(smem + kSeqOffScal);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kSeqOffBar);

  // A CTA pair per KV group: rank r scores chunks [c_begin, c_end) of the
  // group's centroid rows (its half) and stores every key into rank 0's key
  // array; rank 0 then selects.
  const uint32_t rank = cluster_rank();
  const int g = blockIdx.x >> 1, b = g / Hkv, kvh = g % Hkv, G = Hq / Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nchunks = (C + kSeqChunk - 1) / kSeqChunk;
  const int half = (nchunks + 1) / 2;
  const int c_begin = min(nchunks, (int)rank * half), c_end = min(nchunks, c_begin + half);
  const int nmine = c_end - c_begin;
  const unsigned char* cg = reinterpret_cast<const unsigned char*>(cent + (size_t)g * C * kHeadDim);

  // This CTA's centroid rows stream through kSeqStages shared-memory stages by
  // bulk copy (i: this CTA's chunk count, chunk = c_begin + i).
  auto issue = [&](int i) {
    const int st = i % kSeqStages, chunk = c_begin + i;
    const int rows = min(kSeqChunk, C - chunk * kSeqChunk);
    const uint32_t bytes = (uint32_t)rows * kHeadDim * 2;
    mbar_arrive_expect_tx(&bar[st], bytes);
    const unsigned char* src = cg + (size_t)chunk * kSeqChunkBytes;
    unsigned char* dst = smem + (size_t)st * kSeqChunkBytes;
    for (uint32_t o = 0; o < bytes; o += 16384)
      bulk_load(dst + o, src + o, min(16384u, bytes - o), &bar[st], policy_evict_first());
  };
  if (tid == 0) {
    for (int i = 0; i < kSeqStages; ++i) mbar_init(&bar[i], 1);
    fence_barrier_init();
  }
  __syncthreads();
  // the partner runs (its shared memory exists) before the first remote store
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  if (tid == 0)
    for (int i = 0; i < kSeqStages && i < nmine; ++i) issue(i);

  if (tid < kHeadDim) {
    float sum = 0.f;
    for (int h = 0; h < G; ++h)
      sum += __uint_as_float((uint32_t)q[((size_t)b * Hq + kvh * G + h) * kHeadDim + tid] << 16);
    qs[tid] = sum;
  }
  for (int c = tid; c < C; c += kSeqThreads) flag[c] = 0;
  __syncthreads();
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  const uint32_t key0 = map_to(key, 0);  // rank 0's key array

  // ---- scores: 16 lanes per centroid row (8 dims each), 2 rows per warp step
  const int ch = lane & 15;
  float qv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qv[e] = qs[ch * 8 + e];
  for (int i = 0; i < nmine; ++i) {
    const int st = i % kSeqStages, chunk = c_begin + i;
    // an expired wait ends the loop for the whole CTA at once (block barriers follow)
    if (__syncthreads_or(!mbar_wait_bounded(&bar[st], (i / kSeqStages) & 1, nullptr))) break;
    const unsigned char* sc = smem + (size_t)st * kSeqChunkBytes;
    const int rows = min(kSeqChunk, C - chunk * kSeqChunk);
#pragma unroll 4
    for (int rb = warp * 2; rb < rows; rb += (kSeqThreads / 32) * 2) {  // warp-uniform bound
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
      if (valid && ch == 0)
        st_cluster_u32(key0 + 4u * (uint32_t)(chunk * kSeqChunk + r), seq_score_key(acc));
    }
    __syncthreads();  // stage st fully read
    if (tid == 0 && i + kSeqStages < nmine) issue(i + kSeqStages);
  }
  // every key of both halves is in rank 0's array (release / acquire at
  // cluster scope); rank 1 is done
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
  if (rank != 0) return;

  // the token ranges of this thread's clusters, loaded while the selection runs
  const int per = (C + kSeqThreads - 1) / kSeqThreads;  // clusters per thread (<= 8)
  const int c0 = tid * per;
  const int* og = off + (size_t)g * (C + 1);
  int tok[kSeqMaxClusters / kSeqThreads + 1];
#pragma unroll
  for (int i = 0; i <= kSeqMaxClusters / kSeqThreads; ++i)
    tok[i] = (i <= per && c0 + i <= C) ? og[c0 + i] : 0;

  // ---- radix select: the k-th largest key T, 8 bits at a time from the top
  uint32_t prefix = 0, pmask = 0;
  int kk = k;  // rank still to find below the fixed prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSeqThreads) hist[i] = 0;
    __syncthreads();
    for (int c = tid; c < C; c += kSeqThreads) {
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
  int nties = 0;
  for (int c = c0; c < c0 + per && c < C; ++c) nties += (key[c] == T);
  int tot = 0;
  int tie_rank = seq_block_scan(nties, wsum, &tot);
  int cnt = 0;
  for (int c = c0; c < c0 + per && c < C; ++c) {
    const uint32_t kc = key[c];
    int f = kc > T;
    if (kc == T) f = (tie_rank++ < kk);
    flag[c] = (unsigned char)f;
    cnt += f;
  }

  // ---- compact in ascending id order
  int pos = seq_block_scan(cnt, wsum, &tot);
  const size_t ob = (size_t)g * k;
#pragma unroll
  for (int i = 0; i < kSeqMaxClusters / kSeqThreads; ++i) {
    const int c = c0 + i;
    if (i < per && c < C && flag[c]) {
      ids[ob + pos] = c;
      ss[ob + pos] = tok[i];
      se[ob + pos] = tok[i + 1];
      ++pos;
    }
  }
}


struct SelParams {
  const uint16_t* q;     // bf16 [B][Hq][128]
  const uint16_t* cent;  // bf16 [Hkv][C][128], shared by every request
  const int* off;        // [Hkv][C + 1]
  int B, Hq, Hkv, C, k;
  int S;                 // CTAs (and requests) per cluster
  int* ids;
  int* ss;
  int* se;
};

// Order-preserving map of an fp32 score to an unsigned key.
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Arrive on an mbarrier of another CTA of the cluster; release at cluster scope
// orders this thread's earlier (remote) shared-memory stores before it.
__device__ __forceinline__ void arrive_remote(uint32_t bar_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_addr) : "memory");
}
__device__ __forceinline__ bool try_wait_acq_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Block-wide exclusive prefix of per-thread counts (threads own contiguous
// runs in index order); returns the thread's offset, the total in *total.
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
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) {
    if (w < warp) base += wsum[w];
    tot += wsum[w];
  }
  __syncthreads();
  *total = tot;
  return base + incl - cnt;
}

// Top-k of the C keys in shared memory (the k largest, ties to the lower
// index), written ascending to ids / ss / se with the ranges from `og`.
__device__ void topk_write(const uint32_t* key, int C, int k, int* hist, int* wsum, int* scal,
                           const int* og, int* ids, int* ss, int* se) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint32_t prefix = 0, pmask = 0;
  int kk = k;             // rank still to find among the keys matching the prefix
  bool ge_rule = false;   // the boundary digit's keys are all kept: select key >= prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0;
    __syncthreads();
    for (int c0 = warp * 32; c0 < C; c0 += kSelThreads) {  // warp-uniform bound
      const int c = c0 + lane;
      const uint32_t kc = c < C ? key[c] : 0u;
      const bool in = c < C && (kc & pmask) == prefix;
      const int d = in ? (int)((kc >> shift) & 0xFFu) : 256 + lane;  // unique dummy when out
      const uint32_t peers = __match_any_sync(0xffffffffu, d);
      if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[d], __popc(peers));
    }
    __syncthreads();
    if (warp == 0) {  // bins from the top: find the digit holding rank kk
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
            scal[0] = 255 - (lane * 8 + j);  // digit
            scal[1] = kk - before;           // rank within that digit
            scal[2] = cnt[j];                // keys with that digit
          }
          before += cnt[j];
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)scal[0] << shift;
    pmask |= 0xFFu << shift;
    kk = scal[1];
    const bool all_taken = scal[2] == kk;
    __syncthreads();
    if (all_taken) {
      ge_rule = true;
      break;
    }
  }
  const uint32_t T = prefix;  // ge_rule: keep key >= T; else keep keys above T plus kk ties

  // flags in registers: thread t owns ids [t * per, (t + 1) * per)
  const int per = (C + kSelThreads - 1) / kSelThreads;  // <= 8
  const int c0 = tid * per;
  int tie_rank = 0;
  if (!ge_rule) {
    int nties = 0;
    for (int c = c0; c < c0 + per && c < C; ++c) nties += (key[c] == T);
    int tot = 0;
    tie_rank = block_exclusive_scan(nties, wsum, &tot);
  }
  uint32_t fl = 0;
  int cnt = 0;
  for (int i = 0; i < per; ++i) {
    const int c = c0 + i;
    if (c >= C) break;
    const uint32_t kc = key[c];
    int f;
    if (ge_rule) {
      f = kc >= T;
    } else {
      f = kc > T;
      if (kc == T) f = (tie_rank++ < kk);
    }
    fl |= (uint32_t)f << i;
    cnt += f;
  }
  int tot = 0;
  int pos = block_exclusive_scan(cnt, wsum, &tot);
  for (int i = 0; i < per; ++i) {
    if ((fl >> i) & 1u) {
      const int c = c0 + i;
      ids[pos] = c;
      ss[pos] = og[c];
      se[pos] = og[c + 1];
      ++pos;
    }
  }
}

__global__ void __launch_bounds__(kSelThreads, 1) select_kernel(const SelParams p) {
  constexpr int QM = kSelMaxQ;  // most queries a CTA scores
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t* key = reinterpret_cast<uint32_t*>(smem + kOffKeys);
  float* qs = reinterpret_cast<float*>(smem + kOffQ);
  int* hist = reinterpret_cast<int*>(smem + kOffHist);
  int* wsum = reinterpret_cast<int*>(smem + kOffWsum);
  int* scal = reinterpret_cast<int*>(smem + kOffScal);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);  // [stages] ring, [1] gather

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = p.S;
  const uint32_t rank = cluster_rank();
  const int kvh = blockIdx.y, G = p.Hq / p.Hkv;
  // the requests this cluster serves; they share KV head kvh's centroids
  const int b0 = blockIdx.z * S, nq = min(S, p.B - b0), cset = kvh;
  const int r0 = (int)(((long long)rank * p.C) / S), r1 = (int)(((long long)(rank + 1) * p.C) / S);
  const int rows = r1 - r0;
  const int nst = (rows + kStageRows - 1) / kStageRows;
  const unsigned char* src0 =
      reinterpret_cast<const unsigned char*>(p.cent + ((size_t)cset * p.C + r0) * kHeadDim);
  const bool owner = (int)rank < nq;  // this CTA owns request rank's selection

  auto issue = [&](int chunk) {
    const int st = chunk % kSelStages;
    const int n = min(kStageRows, rows - chunk * kStageRows);
    const uint32_t bytes = (uint32_t)n * kRowBytes;
    mbar_arrive_expect_tx(&bar[st], bytes);
    const unsigned char* src = src0 + (size_t)chunk * kStageBytes;
    unsigned char* dst = smem + (size_t)st * kStageBytes;
    for (uint32_t o = 0; o < bytes; o += 16384)
      bulk_load(dst + o, src + o, min(16384u, bytes - o), &bar[st], policy_evict_first());
  };
  if (tid == 0) {
    for (int i = 0; i < kSelStages; ++i) mbar_init(&bar[i], 1);
    mbar_init(&bar[kSelStages], S);  // one arrival per CTA of the cluster
    fence_barrier_init();
  }
  __syncthreads();
  // every thread marks the cluster barrier once this CTA's mbarriers are ready;
  // the wait before the first remote access ends once every CTA has done so
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  if (tid == 0)
    for (int i = 0; i < kSelStages && i < nst; ++i) issue(i);

  // summed query heads of every request served, fp32 (bf16 inputs are exact)
  for (int i = tid; i < nq * kHeadDim; i += kSelThreads) {
    const int j = i / kHeadDim, dd = i % kHeadDim;
    const uint16_t* qr = p.q + ((size_t)(b0 + j) * p.Hq + (size_t)kvh * G) * kHeadDim + dd;
    float sum = 0.f;
    for (int h = 0; h < G; ++h) sum += __uint_as_float((uint32_t)qr[(size_t)h * kHeadDim] << 16);
    qs[i] = sum;
  }
  __syncthreads();

  // ---- scores: 16 lanes per centroid row (8 dims each), 2 rows per warp step
  const int ch = lane & 15;
  float qv[QM][8];
#pragma unroll
  for (int j = 0; j < QM; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) qv[j][e] = j < nq ? qs[j * kHeadDim + ch * 8 + e] : 0.f;
  // remote key slots: query j's owner is rank j
  uint32_t kaddr[QM];
#pragma unroll
  for (int j = 0; j < QM; ++j) kaddr[j] = map_to(key, (uint32_t)min(j, S - 1));
  bool ok = true;
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  for (int chunk = 0; chunk < nst; ++chunk) {
    const int st = chunk % kSelStages;
    // an expired wait ends the loop for the whole CTA at once (block barriers follow)
    if (__syncthreads_or(!mbar_wait_bounded(&bar[st], (chunk / kSelStages) & 1, nullptr))) {
      ok = false;
      break;
    }
    const unsigned char* sc = smem + (size_t)st * kStageBytes;
    const int n = min(kStageRows, rows - chunk * kStageRows);
    for (int rb = warp * 2; rb < n; rb += kSelWarps * 2) {  // warp-uniform bound
      const int r = rb + (lane >> 4);
      const bool valid = r < n;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (valid) w = *reinterpret_cast<const uint4*>(sc + (size_t)r * kRowBytes + ch * 16);
      const float kf[8] = {__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u),
                           __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u),
                           __uint_as_float(w.z << 16), __uint_as_float(w.z & 0xFFFF0000u),
                           __uint_as_float(w.w << 16), __uint_as_float(w.w & 0xFFFF0000u)};
      const int c = r0 + chunk * kStageRows + r;
#pragma unroll
      for (int j = 0; j < QM; ++j) {
        if (j >= nq) break;  // uniform across the CTA
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc = fmaf(qv[j][e], kf[e], acc);
        acc += __shfl_xor_sync(0xffffffffu, acc, 8);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        if (valid && ch == j) st_cluster_u32(kaddr[j] + 4u * (uint32_t)c, score_key(acc));
      }
    }
    __syncthreads();  // stage st fully read
    if (tid == 0 && chunk + kSelStages < nst) issue(chunk + kSelStages);
  }
  // this CTA's keys are stored: arrive on every owner's gather barrier
  __syncthreads();
  if (tid < nq) arrive_remote(map_to(&bar[kSelStages], (uint32_t)tid));
  if (!owner) return;  // (nothing reads this CTA's shared memory)

  bool got = false;
  {
    const uint64_t t0 = globaltimer();
    while (!(got = try_wait_acq_cluster(&bar[kSelStages], 0)))
      if (globaltimer() - t0 > 4 * kWaitLimitNs) break;
  }
  const int b = b0 + (int)rank;
  const size_t ob = ((size_t)b * p.Hkv + kvh) * p.k;
  const int* og = p.off + (size_t)cset * (p.C + 1);
  if (!ok || !got) {  // a bounded wait expired: no selection (empty ranges)
    for (int i = tid; i < p.k; i += kSelThreads) {
      p.ids[ob + i] = -1;
      p.ss[ob + i] = 0;
      p.se[ob + i] = 0;
    }
    return;
  }
  topk_write(key, p.C, p.k, hist, wsum, scal, og, p.ids + ob, p.ss + ob, p.se + ob);
}

}  // namespace

// Requests (and CTAs) per cluster of the shared-centroid kernel: up to 8.
int select_cluster_size(int B) { return B < 1 ? 1 : (B < kSelMaxQ ? B : kSelMaxQ); }

int launch_select(const uint16_t* q, const uint16_t* cent, const int* off, int B, int Hq, int Hkv,
                  int C, int k, int shared, int* ids, int* ss, int* se, void* stream) {
  static std::atomic<bool> attr_set[64][2];  // per device; racing first calls only repeat the set-up
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
  if (!shared) {  // a CTA pair per KV group
    if (!attr_set[dev][0]) {
      cudaError_t e = cudaFuncSetAttribute(select_seq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kSeqSmem);
      if (e != cudaSuccess) return (int)e;
      attr_set[dev][0] = true;
    }
    select_seq_kernel<<<2 * B * Hkv, kSeqThreads, kSeqSmem, static_cast<cudaStream_t>(stream)>>>(
        q, cent, off, Hq, Hkv, C, k, ids, ss, se);
    return (int)cudaGetLastError();
  }
  SelParams p{};
  p.q = q;
  p.cent = cent;
  p.off = off;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.C = C;
  p.k = k;
  p.S = select_cluster_size(B);
  p.ids = ids;
  p.ss = ss;
  p.se = se;
  auto kern = select_kernel;
  if (!attr_set[dev][1]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSelSmem);
    if (e != cudaSuccess) return (int)e;
    attr_set[dev][1] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.S, Hkv, (B + p.S - 1) / p.S);
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.dynamicSmemBytes = kSelSmem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace skv
