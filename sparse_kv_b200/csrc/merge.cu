// merge.cu -- exact log-sum-exp merge of attention partials
// ("Pulsar Attention" Phase 2: per-shard local attention combined by the
// online-softmax merge into the exact global result).
//
// One warp per output row; lane j owns dims 4j.. (float4), looping for
// head_dim > 128.  HBM-bound: reads S*(d+1) floats and writes d+1 per row.
#include "common.cuh"
#include "decode.cuh"

namespace skv {
namespace {

constexpr int kMergeWarps = 8;

__global__ void __launch_bounds__(kMergeWarps * 32) merge_kernel(const float* __restrict__ o,
                                                               const float* __restrict__ l, int S,
                                                               int N, int d, float* __restrict__ out,
                                                               float* __restrict__ lse) {
  const int row = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, l[(size_t)s * N + row]);
  if (M == -INFINITY) {
    for (int j = lane * 4; j < d; j += 128)
      *reinterpret_cast<float4*>(out + (size_t)row * d + j) = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane == 0) lse[row] = -INFINITY;
    return;
  }
  float4 acc[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
  float W = 0.f;
  for (int s = 0; s < S; ++s) {
    const float w = expf(l[(size_t)s * N + row] - M);  // 0 for an empty partial
    W += w;
    if (w == 0.f) continue;
    const float* src = o + ((size_t)s * N + row) * d;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = lane * 4 + u * 128;
      if (j < d) {
        const float4 v = *reinterpret_cast<const float4*>(src + j);
        acc[u].x += w * v.x;
        acc[u].y += w * v.y;
        acc[u].z += w * v.z;
        acc[u].w += w * v.w;
      }
    }
  }
  const float inv = 1.f / W;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = lane * 4 + u * 128;
    if (j < d)
      *reinterpret_cast<float4*>(out + (size_t)row * d + j) =
          make_float4(acc[u].x * inv, acc[u].y * inv, acc[u].z * inv, acc[u].w * inv);
  }
  if (lane == 0) lse[row] = M + logf(W);
}

}  // namespace

int launch_merge(const float* o_parts, const float* lse_parts, int S, int N, int d, float* out,
                 float* lse, void* stream) {
  if (N == 0) return 0;
  const int blocks = (N + kMergeWarps - 1) / kMergeWarps;
  merge_kernel<<<blocks, kMergeWarps * 32, 0, static_cast<cudaStream_t>(stream)>>>(
      o_parts, lse_parts, S, N, d, out, lse);
  return (int)cudaGetLastError();
}

}  // namespace skv

// ---------------------------------------------------------------------------
// Merge of the decode kernels' partial records.  Row (b, h) of group
// g = b*Hkv + h/G collects the records of every piece of g: persistent
// schedule -> slots c + g for the CTAs c whose tile share meets g's tiles
// [T_g, T_g + n_g); ART -> the chunks of g up to the one where the row's head
// stopped.  (The split schedule merges inside decode_kernel.)  Each record holds
// (O unnormalised, m in base 2, l, tiles); the merge is the same exact
// online-softmax combination as above, in base 2.
// ---------------------------------------------------------------------------
namespace skv {
namespace {

// One CTA of kMergeWarps warps per output row.  Records are spread over all
// threads for the per-record scalars (m, l, tiles) and over the warps for the
// O vectors (lane j owns dims 4j..4j+3), so many independent loads are in
// flight; the warps' partial sums are combined through shared memory.
__global__ void __launch_bounds__(kMergeWarps * 32) merge_records_kernel(const DecodeParams p, int G,
                                                                        int NW) {
  extern __shared__ float fw[];  // [nrec] weights
  __shared__ float red[kMergeWarps][2];
  __shared__ float4 part[kMergeWarps][32];
  const int row = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int NT = kMergeWarps * 32;
  const int b = row / p.Hq, h = row % p.Hq, kvh = h / G, gh = h % G;
  const int g = b * p.Hkv + kvh;
  int s0 = 0, s1 = -1;  // slot range [s0, s1]
  long long T = 0, P = p.n_ctas;
  int art_used = 0;
  if (p.sched == SCHED_ART) {
    const int groups = p.B * p.Hkv;
    const int* stop_chunk = p.art_ctl + 4;
    const int* consumed = stop_chunk + groups + (size_t)groups * p.art_maxc;
    const int* head_stop = consumed + (size_t)groups * G;
    int L = p.seq_lens[b];
    if (L < 0 || L > p.max_seq_len) L = 0;
    int nch = (art_positions(p, L) + p.art_chunk - 1) / p.art_chunk;
    const int sc = head_stop[(size_t)g * G + gh];  // the head's stop chunk + 1
    if (sc != 0 && sc < nch) nch = sc;
    s0 = g * p.art_maxc;
    s1 = s0 + nch - 1;
    art_used = consumed[(size_t)g * G + gh];
  } else if (p.sched == SCHED_PERSISTENT) {
    T = p.ws_hdr[0];
    const int pb = p.ws_hdr[1 + b], pb1 = p.ws_hdr[2 + b];
    const int nt = (pb1 - pb) / p.Hkv;
    if (nt > 0 && T > 0) {
      const long long Tg = pb + (long long)kvh * nt;
      s0 = (int)(((Tg + 1) * P - 1) / T) + g;
      s1 = (int)(((Tg + nt) * P - 1) / T) + g;
    }
  }
  const int nrec = (s1 - s0 + 1) * NW;  // record r: slot s0 + r / NW, warp r % NW
  auto rec_ptr = [&](int r) {
    return p.ws_rec + (((size_t)(s0 + r / NW) * NW + (r % NW)) * G + gh) * kRecFloats;
  };
  // pass 1: scalars of every record; block max of m and sum of tiles
  float M = -INFINITY;
  int tiles = 0;
  for (int r = tid; r < nrec; r += NT) {
    float m = -INFINITY;
    bool valid = true;
    if (p.sched == SCHED_PERSISTENT) {  // a CTA whose share of tiles is empty wrote nothing
      const long long c = s0 + r / NW - g;
      valid = (c * T) / P != ((c + 1) * T) / P;
    }
    if (valid) {
      const float4 ml = *reinterpret_cast<const float4*>(rec_ptr(r) + 128);  // m, l, tiles
      if (ml.y > 0.f) m = ml.x;
      if (r % NW == 0) tiles += (int)ml.z;
    }
    fw[r] = m;  // -inf for an empty or unwritten record; turned into a weight below
    M = fmaxf(M, m);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    tiles += __shfl_xor_sync(0xffffffffu, tiles, o);
  }
  if (lane == 0) {
    red[warp][0] = M;
    red[warp][1] = __int_as_float(tiles);
  }
  __syncthreads();
  M = -INFINITY;
  tiles = 0;
#pragma unroll
  for (int w = 0; w < kMergeWarps; ++w) {
    M = fmaxf(M, red[w][0]);
    tiles += __float_as_int(red[w][1]);
  }
  // pass 2: weights f_r = 2^(m_r - M) and W = sum f_r l_r (l re-read from the record)
  float W = 0.f;
  for (int r = tid; r < nrec; r += NT) {
    const float m = fw[r];
    float f = 0.f;
    if (m != -INFINITY) {
      f = exp2f(m - M);
      W += f * rec_ptr(r)[129];
    }
    fw[r] = f;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
  __syncthreads();
  if (lane == 0) red[warp][0] = W;
  __syncthreads();
  W = 0.f;
#pragma unroll
  for (int w = 0; w < kMergeWarps; ++w) W += red[w][0];
  // pass 3: O = sum f_r O_r, warp w takes records w, w + kMergeWarps, ... (8 in flight)
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r0 = warp; r0 < nrec; r0 += kMergeWarps * 8) {
    float4 o[8];
    float f[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int r = r0 + q * kMergeWarps;
      f[q] = (r < nrec) ? fw[r] : 0.f;
      o[q] = (f[q] > 0.f) ? *reinterpret_cast<const float4*>(rec_ptr(r) + lane * 4)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      acc.x += f[q] * o[q].x;
      acc.y += f[q] * o[q].y;
      acc.z += f[q] * o[q].z;
      acc.w += f[q] * o[q].w;
    }
  }
  part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) {
      s.x += part[w][lane].x;
      s.y += part[w][lane].y;
      s.z += part[w][lane].z;
      s.w += part[w][lane].w;
    }
    const float inv = (W > 0.f) ? 1.f / W : 0.f;
    *reinterpret_cast<float4*>(p.out + (size_t)row * kHeadDim + lane * 4) =
        make_float4(s.x * inv, s.y * inv, s.z * inv, s.w * inv);
    if (lane == 0) {
      p.lse[row] = (W > 0.f) ? (M + log2f(W)) * 0.6931471805599453f : -INFINITY;
      if (p.blocks_consumed) p.blocks_consumed[row] = (p.sched == SCHED_ART) ? art_used : tiles;
    }
  }
}

}  // namespace

int launch_merge_records(const DecodeParams& p, int G, void* stream) {
  const int N = p.B * p.Hq;
  if (N == 0) return 0;
  // records per row: pieces of one group (<= all persistent CTAs, or the splits) x warps
  if (p.sched != SCHED_PERSISTENT && p.sched != SCHED_ART) return (int)cudaErrorInvalidValue;
  const int max_slots = (p.sched == SCHED_PERSISTENT) ? p.n_ctas : p.art_maxc;
  const size_t smem = (size_t)max_slots * p.rec_nw * sizeof(float);
  if (smem > 200 * 1024) return (int)cudaErrorInvalidConfiguration;
  static std::atomic<bool> attr_set[64];  // per device; racing first calls only repeat the set-up
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(merge_records_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return (int)e;
    attr_set[dev] = true;
  }
  merge_records_kernel<<<N, kMergeWarps * 32, smem, static_cast<cudaStream_t>(stream)>>>(
      p, G, p.rec_nw);
  return (int)cudaGetLastError();
}

}  // namespace skv
