// skvgen/device.cu -- device side of the seeded input generator (C ABI).
//
// Fills GPU buffers (the paged K/V pool, q, centroids) with exactly the values
// host.c produces in logical layout, so large workloads never cross PCIe.
// Test infrastructure only: the attention library does not link this file.
#include <cuda_runtime.h>
#include <stdint.h>

#include "core.h"

namespace {

__global__ void k_normal(uint64_t key, uint64_t base, uint64_t n, uint16_t* out) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = skvg_normal_bf16(key, base + i);
}

// One thread per KV group: same sequential fp64 steps as skvg_host_qhat.
__global__ void k_qhat(const uint16_t* q, int B, int Tq, int Hq, int Hkv, int d, double* qhat) {
  int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= B * Hkv) return;
  int b = g / Hkv, kvh = g % Hkv, G = Hq / Hkv;
  const uint16_t* qg = q + ((uint64_t)b * Tq * Hq + (uint64_t)kvh * G) * d;  // token 0
  double* o = qhat + (uint64_t)g * d;
  double ss = 0.0;
  for (int j = 0; j < d; ++j) {
    double s = 0.0;
    for (int h = 0; h < G; ++h) s = SKVG_DADD(s, skvg_bf16_to_f64(qg[h * d + j]));
    o[j] = s;
  }
  for (int j = 0; j < d; ++j) ss = SKVG_DADD(ss, SKVG_DMUL(o[j], o[j]));
  double nrm = SKVG_DSQRT(ss);
  for (int j = 0; j < d; ++j) o[j] = nrm > 0.0 ? SKVG_DDIV(o[j], nrm) : 0.0;
}

// Element (g, t, j) of the logical K/V, written to page block_table[b][t/bs].
__global__ void k_kv_paged(uint64_t kk, uint64_t kv, uint64_t kh, int B, int Hkv, int d,
                           uint64_t Lmax, const int* seq_lens, const int* block_table,
                           int max_blocks, int bs, const double* qhat, uint16_t* k_pool,
                           uint16_t* v_pool) {
  uint64_t n = (uint64_t)B * Hkv * Lmax * d;
  for (uint64_t e = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; e < n;
       e += (uint64_t)gridDim.x * blockDim.x) {
    uint64_t j = e % d;
    uint64_t t = (e / d) % Lmax;
    uint64_t g = e / ((uint64_t)d * Lmax);
    int b = (int)(g / Hkv), kvh = (int)(g % Hkv);
    if (t >= (uint64_t)seq_lens[b]) continue;
    int page = block_table[(uint64_t)b * max_blocks + t / bs];
    if (page < 0) continue;
    uint64_t dst = (((uint64_t)page * Hkv + kvh) * bs + t % bs) * d + j;
    uint64_t c = (g * Lmax + t) * d + j;
    if (k_pool) {
      uint16_t k = skvg_normal_bf16(kk, c);
      if (qhat) {
        double coef = (t == 0) ? 6.0 : (skvg_is_heavy(kh, g, Lmax, t) ? 4.0 : 0.0);
        if (coef != 0.0) k = skvg_shift_bf16(k, coef, qhat[g * d + j]);
      }
      k_pool[dst] = k;
    }
    if (v_pool) v_pool[dst] = skvg_normal_bf16(kv, c);
  }
}

__global__ void k_mix_count(uint64_t ka, int G, uint64_t Lmax, uint64_t L, uint32_t c_log2,
                            int* off) {
  uint64_t n = (uint64_t)G * L;
  uint32_t C = 1u << c_log2;
  for (uint64_t e = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; e < n;
       e += (uint64_t)gridDim.x * blockDim.x) {
    uint64_t g = e / L, i = e % L;
    atomicAdd(&off[g * (C + 1) + skvg_component(ka, g, Lmax, i, c_log2) + 1], 1);
  }
}

__global__ void k_mix_scan(int G, uint32_t c_log2, int* off) {
  int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= G) return;
  uint32_t C = 1u << c_log2;
  int* o = off + (uint64_t)g * (C + 1);
  for (uint32_t c = 0; c < C; ++c) o[c + 1] += o[c];
}

__global__ void k_mix_keys(uint64_t kc, uint64_t kk, int Hkv, int d, uint64_t Lmax, uint64_t L,
                           uint32_t c_log2, const int* off, const int* block_table, int max_blocks,
                           int bs, int G, uint16_t* k_pool) {
  uint32_t C = 1u << c_log2;
  uint64_t n = (uint64_t)G * L * d;
  for (uint64_t e = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; e < n;
       e += (uint64_t)gridDim.x * blockDim.x) {
    uint64_t j = e % d;
    uint64_t t = (e / d) % L;
    uint64_t g = e / ((uint64_t)d * L);
    const int* o = off + g * (C + 1);
    // largest c with o[c] <= t  (clusters may be empty)
    uint32_t lo = 0, hi = C;  // invariant: o[lo] <= t < o[hi]
    while (hi - lo > 1) {
      uint32_t mid = (lo + hi) >> 1;
      if ((uint64_t)o[mid] <= t) lo = mid; else hi = mid;
    }
    uint16_t center = skvg_normal_bf16(kc, (g * C + lo) * d + j);
    float nz = skvg_normal(kk, (g * Lmax + t) * d + j);
    int b = (int)(g / Hkv), kvh = (int)(g % Hkv);
    int page = block_table[(uint64_t)b * max_blocks + t / bs];
    if (page < 0) continue;
    k_pool[(((uint64_t)page * Hkv + kvh) * bs + t % bs) * d + j] = skvg_mixture_key(center, nz);
  }
}

__global__ void k_mix_centroids(uint64_t kc, uint64_t kk, int d, uint64_t Lmax, uint32_t c_log2,
                                const int* off, int G, uint16_t* centroids) {
  uint32_t C = 1u << c_log2;
  uint64_t n = (uint64_t)G * C * d;
  for (uint64_t e = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; e < n;
       e += (uint64_t)gridDim.x * blockDim.x) {
    uint64_t j = e % d;
    uint64_t c = (e / d) % C;
    uint64_t g = e / ((uint64_t)d * C);
    const int* o = off + g * (C + 1);
    uint16_t center = skvg_normal_bf16(kc, (g * C + c) * d + j);
    double sum = 0.0;
    for (int t = o[c]; t < o[c + 1]; ++t) {
      float nz = skvg_normal(kk, (g * Lmax + (uint64_t)t) * d + j);
      sum = SKVG_DADD(sum, skvg_bf16_to_f64(skvg_mixture_key(center, nz)));
    }
    int sz = o[c + 1] - o[c];
    centroids[e] = sz > 0 ? skvg_f64_to_bf16(SKVG_DDIV(sum, (double)sz)) : center;
  }
}

// Block summaries: element (b, kvh, j, dim) = bf16( fp64 mean of the keys of
// logical block j of sequence b, KV head kvh ); blocks past the sequence are 0.
__global__ void k_block_means(const uint16_t* k_pool, const int* block_table, const int* seq_lens,
                              int B, int Hkv, int d, int max_blocks, int bs, uint16_t* out) {
  uint64_t n = (uint64_t)B * Hkv * max_blocks * d;
  for (uint64_t e = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; e < n;
       e += (uint64_t)gridDim.x * blockDim.x) {
    uint64_t j = e % d;
    uint64_t blk = (e / d) % max_blocks;
    uint64_t kvh = (e / ((uint64_t)d * max_blocks)) % Hkv;
    uint64_t b = e / ((uint64_t)d * max_blocks * Hkv);
    int L = seq_lens[b];
    int t0 = (int)blk * bs, t1 = t0 + bs < L ? t0 + bs : L;
    int page = block_table[b * max_blocks + blk];
    if (t1 <= t0 || page < 0) {
      out[e] = 0;
      continue;
    }
    double sum = 0.0;
    for (int t = t0; t < t1; ++t)
      sum = SKVG_DADD(sum, skvg_bf16_to_f64(k_pool[(((uint64_t)page * Hkv + kvh) * bs + (t - t0)) * d + j]));
    out[e] = skvg_f64_to_bf16(SKVG_DDIV(sum, (double)(t1 - t0)));
  }
}

inline int grid_for(uint64_t n) {
  uint64_t g = (n + 255) / 256;
  return (int)(g > 148ull * 64 ? 148ull * 64 : (g == 0 ? 1 : g));
}

}  // namespace

extern "C" {

int skvg_dev_normal_bf16(uint64_t seed, uint32_t stream, uint32_t layer, uint64_t base, uint64_t n,
                         uint16_t* out, cudaStream_t st) {
  if (n == 0) return 0;
  k_normal<<<grid_for(n), 256, 0, st>>>(skvg_key(seed, stream, layer), base, n, out);
  return (int)cudaGetLastError();
}

int skvg_dev_qhat(const uint16_t* q, int B, int Tq, int Hq, int Hkv, int d, double* qhat,
                  cudaStream_t st) {
  int G = B * Hkv;
  k_qhat<<<(G + 63) / 64, 64, 0, st>>>(q, B, Tq, Hq, Hkv, d, qhat);
  return (int)cudaGetLastError();
}

int skvg_dev_kv_paged(uint64_t seed, uint32_t layer, int B, int Hkv, int d, uint64_t Lmax,
                      const int* seq_lens, const int* block_table, int max_blocks, int bs,
                      const double* qhat, uint16_t* k_pool, uint16_t* v_pool, cudaStream_t st) {
  uint64_t n = (uint64_t)B * Hkv * Lmax * d;
  if (n == 0) return 0;
  k_kv_paged<<<grid_for(n), 256, 0, st>>>(
      skvg_key(seed, SKVG_S_K, layer), skvg_key(seed, SKVG_S_V, layer),
      skvg_key(seed, SKVG_S_HEAVY, layer), B, Hkv, d, Lmax, seq_lens, block_table, max_blocks, bs,
      qhat, k_pool, v_pool);
  return (int)cudaGetLastError();
}

// off: device int [B*Hkv][C+1], zeroed here.  Keys go to k_pool through the
// block table; values are filled separately with skvg_dev_kv_paged(k_pool=NULL).
int skvg_dev_mixture(uint64_t seed, uint32_t layer, int B, int Hkv, int d, uint64_t Lmax, uint64_t L,
                     uint32_t c_log2, const int* block_table, int max_blocks, int bs,
                     uint16_t* k_pool, int* off, uint16_t* centroids, cudaStream_t st) {
  int G = B * Hkv;
  uint32_t C = 1u << c_log2;
  cudaError_t e = cudaMemsetAsync(off, 0, sizeof(int) * (size_t)G * (C + 1), st);
  if (e != cudaSuccess) return (int)e;
  uint64_t ka = skvg_key(seed, SKVG_S_ASSIGN, layer);
  uint64_t kc = skvg_key(seed, SKVG_S_CENTER, layer);
  uint64_t kk = skvg_key(seed, SKVG_S_K, layer);
  k_mix_count<<<grid_for((uint64_t)G * L), 256, 0, st>>>(ka, G, Lmax, L, c_log2, off);
  k_mix_scan<<<(G + 63) / 64, 64, 0, st>>>(G, c_log2, off);
  if (k_pool)
    k_mix_keys<<<grid_for((uint64_t)G * L * d), 256, 0, st>>>(kc, kk, Hkv, d, Lmax, L, c_log2, off,
                                                              block_table, max_blocks, bs, G,
                                                              k_pool);
  if (centroids)
    k_mix_centroids<<<grid_for((uint64_t)G * C * d), 256, 0, st>>>(kc, kk, d, Lmax, c_log2, off,
                                                                   G, centroids);
  return (int)cudaGetLastError();
}

int skvg_dev_block_means(const uint16_t* k_pool, const int* block_table, const int* seq_lens, int B,
                         int Hkv, int d, int max_blocks, int bs, uint16_t* out, cudaStream_t st) {
  uint64_t n = (uint64_t)B * Hkv * max_blocks * d;
  if (n == 0) return 0;
  k_block_means<<<grid_for(n), 256, 0, st>>>(k_pool, block_table, seq_lens, B, Hkv, d, max_blocks, bs, out);
  return (int)cudaGetLastError();
}

}  // extern "C"
