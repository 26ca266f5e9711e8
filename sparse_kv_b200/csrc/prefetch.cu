// prefetch.cu -- lookahead selection and prefetch of KV blocks from host
// memory ("SparDA", technical summary section 2: a per-layer Forecast
// projection F_l, one head per GQA group, predicts the top-k blocks layer l+1
// needs; while layer l runs, a fixed set of CTAs pulls those blocks from CPU
// memory into the GPU through unified virtual addressing, so the transfer
// overlaps the current layer's work).
//
//   forecast_kernel   f[b][kvh] = bf16( W[kvh]^T x[b][kvh] ): one CTA per
//                     (b, kvh), thread j accumulates output dim j in fp32 over
//                     the input dims in order (fused multiply-adds), rounded
//                     to bf16 once.  The block choice itself is the
//                     centroid-selection kernel with f as the query and the
//                     layer's block summaries as the centroids.
//   gather_kernel     a fixed grid of CTAs walks the (request, KV head, slot)
//                     items of the chosen blocks; each CTA copies a block's K
//                     and V rows (2 x 16 KiB) from the page-locked host pool,
//                     read through its device-mapped address with 16-byte
//                     loads kept in flight, into slot i of request b's pages
//                     of the device cache, and writes the token range the slot
//                     holds, so that attn_decode's segment traversal attends
//                     exactly the chosen blocks.
#include <cuda_bf16.h>

#include "common.cuh"
#include "decode.cuh"

namespace skv {
namespace {

// Small CTAs (two warps, few registers, no shared memory) fit beside two
// resident CTAs of the decode kernels on the same SM, so the copy overlaps a
// persistent attention kernel whichever starts first.
constexpr int kGatherThreads = 64;
constexpr int kBlockVecs = kTileBytes / 16;  // 16-byte vectors per 16 KiB tile
constexpr int kGatherBatch = 8;              // 16-byte vectors in flight per thread
static_assert(kBlockVecs % (kGatherThreads * kGatherBatch) == 0, "tile split");

__global__ void __launch_bounds__(kHeadDim) forecast_kernel(const uint16_t* __restrict__ x,
                                                            const uint16_t* __restrict__ w, int Hkv,
                                                            uint16_t* __restrict__ f) {
  __shared__ float xs[kHeadDim];
  const int kvh = blockIdx.x, b = blockIdx.y, j = threadIdx.x;
  const size_t row = ((size_t)b * Hkv + kvh) * kHeadDim;
  xs[j] = __uint_as_float((uint32_t)x[row + j] << 16);
  __syncthreads();
  const uint16_t* wk = w + (size_t)kvh * kHeadDim * kHeadDim;  // [in][out]
  float acc = 0.f;
#pragma unroll 8
  for (int i = 0; i < kHeadDim; ++i)
    acc = __fmaf_rn(__uint_as_float((uint32_t)wk[(size_t)i * kHeadDim + j] << 16), xs[i], acc);
  const __nv_bfloat16 h = __float2bfloat16_rn(acc);
  f[row + j] = *reinterpret_cast<const uint16_t*>(&h);
}

struct GatherParams {
  const uint16_t* k_host;  // device-mapped addresses of the host pools [pages][Hkv][64][128]
  const uint16_t* v_host;
  const int* block_table;  // [B][max_blocks]: host pages
  const int* seq_lens;     // [B]
  const int* ids;          // [B][Hkv][k] chosen logical blocks (ascending; -1 = none)
  int B, Hkv, k, max_blocks, num_pages, max_seq_len;
  uint16_t* k_cache;       // [B * k][Hkv][64][128]
  uint16_t* v_cache;
  int* seg_start;          // [B][Hkv][k] token ranges in the cache's coordinates
  int* seg_end;
  uint32_t* status;
};

__device__ __forceinline__ uint4 ld_sys_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// at most 64 registers: 2 warps x 32 x 64 = 4096 registers, which two CTAs of
// the decode kernels (at most 2 x 30720) leave free on an SM
__global__ void __launch_bounds__(kGatherThreads, 16) gather_kernel(const GatherParams p) {
  const long long items = (long long)p.B * p.Hkv * p.k;
  const int tid = threadIdx.x;
  for (long long it = blockIdx.x; it < items; it += gridDim.x) {
    const int slot = (int)(it % p.k);
    const int kvh = (int)((it / p.k) % p.Hkv);
    const int b = (int)(it / ((long long)p.k * p.Hkv));
    int L = p.seq_lens[b];
    if (L < 0 || L > p.max_seq_len) {
      if (tid == 0 && slot == 0 && kvh == 0) dev_error(p.status, SKV_DEV_BAD_SEQLEN);
      L = 0;
    }
    const int nb = (L + kBlock - 1) / kBlock;
    const int j = p.ids[it];  // -1 (nothing chosen) or a block past the sequence: an empty slot
    int n = 0, page = -1;
    if (j >= 0 && j < nb) {
      page = p.block_table[(size_t)b * p.max_blocks + j];
      if (page < 0 || page >= p.num_pages) {
        if (tid == 0) dev_error(p.status, SKV_DEV_BAD_PAGE);
        page = -1;
      } else {
        n = min(kBlock, L - j * kBlock);
      }
    }
    if (tid == 0) {
      p.seg_start[it] = slot * kBlock;
      p.seg_end[it] = slot * kBlock + n;  // empty for no block
    }
    if (page < 0) continue;
    const size_t src = ((size_t)page * p.Hkv + kvh) * (size_t)kBlock * kHeadDim;
    const size_t dst = (((size_t)b * p.k + slot) * p.Hkv + kvh) * (size_t)kBlock * kHeadDim;
    const uint4* ks = reinterpret_cast<const uint4*>(p.k_host + src);
    const uint4* vs = reinterpret_cast<const uint4*>(p.v_host + src);
    uint4* kd = reinterpret_cast<uint4*>(p.k_cache + dst);
    uint4* vd = reinterpret_cast<uint4*>(p.v_cache + dst);
    const int nvec = n * (kRowBytes / 16);  // rows of the block that hold tokens
    for (int t = 0; t < 2; ++t) {             // K rows, then V rows
      const uint4* src4 = (t == 0 ? ks : vs) + tid;
      uint4* dst4 = (t == 0 ? kd : vd) + tid;
      for (int base = 0; base < nvec; base += kGatherThreads * kGatherBatch) {
        uint4 r[kGatherBatch];
#pragma unroll
        for (int u = 0; u < kGatherBatch; ++u)  // all of a batch's loads in flight at once
          if (base + tid + u * kGatherThreads < nvec) r[u] = ld_sys_v4(src4 + base + u * kGatherThreads);
#pragma unroll
        for (int u = 0; u < kGatherBatch; ++u)
          if (base + tid + u * kGatherThreads < nvec) dst4[base + u * kGatherThreads] = r[u];
      }
    }
  }
}

}  // namespace

int launch_forecast(const uint16_t* x, const uint16_t* w, int B, int Hkv, uint16_t* f, void* stream) {
  forecast_kernel<<<dim3(Hkv, B), kHeadDim, 0, static_cast<cudaStream_t>(stream)>>>(x, w, Hkv, f);
  return (int)cudaGetLastError();
}

int launch_gather(const void* k_host, const void* v_host, const int* block_table, const int* seq_lens,
                  const int* ids, int B, int Hkv, int k, int max_blocks, int num_pages, int max_seq_len,
                  void* k_cache, void* v_cache, int* seg_start, int* seg_end, uint32_t* status,
                  int n_ctas, void* stream) {
  GatherParams p{};
  p.k_host = static_cast<const uint16_t*>(k_host);
  p.v_host = static_cast<const uint16_t*>(v_host);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.ids = ids;
  p.B = B;
  p.Hkv = Hkv;
  p.k = k;
  p.max_blocks = max_blocks;
  p.num_pages = num_pages;
  p.max_seq_len = max_seq_len;
  p.k_cache = static_cast<uint16_t*>(k_cache);
  p.v_cache = static_cast<uint16_t*>(v_cache);
  p.seg_start = seg_start;
  p.seg_end = seg_end;
  p.status = status;
  gather_kernel<<<n_ctas, kGatherThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return (int)cudaGetLastError();
}

}  // namespace skv
