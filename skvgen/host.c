/*
 * skvgen/host.c -- host side of the seeded input generator (C ABI).
 *
 * Produces tensors in LOGICAL layout (per KV group, token-major) for the CPU
 * oracle, bit-identical to what device.cu writes into the paged GPU pool.
 * Build: gcc -O2 -fPIC -shared -ffp-contract=off -fopenmp.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "core.h"

uint64_t skvg_host_key(uint64_t seed, uint32_t stream, uint32_t layer) {
  return skvg_key(seed, stream, layer);
}

/* out[i] = bf16 normal sample number (base + i) of tensor (seed, stream, layer). */
void skvg_host_normal_bf16(uint64_t seed, uint32_t stream, uint32_t layer, uint64_t base,
                           uint64_t n, uint16_t* out) {
  uint64_t key = skvg_key(seed, stream, layer);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = skvg_normal_bf16(key, base + (uint64_t)i);
}

/* qhat = unit vector of the sum of the G query heads of one KV group, fp64.
 * q_group: bf16 [G][d] (token 0 of the query, heads kvh*G .. kvh*G+G-1). */
void skvg_host_qhat(const uint16_t* q_group, int G, int d, double* qhat) {
  double ss = 0.0;
  for (int j = 0; j < d; ++j) {
    double s = 0.0;
    for (int g = 0; g < G; ++g) s = SKVG_DADD(s, skvg_bf16_to_f64(q_group[g * d + j]));
    qhat[j] = s;
  }
  for (int j = 0; j < d; ++j) ss = SKVG_DADD(ss, SKVG_DMUL(qhat[j], qhat[j]));
  double nrm = SKVG_DSQRT(ss);
  for (int j = 0; j < d; ++j) qhat[j] = nrm > 0.0 ? SKVG_DDIV(qhat[j], nrm) : 0.0;
}

/* Keys and values of KV group g = b*Hkv + kvh, tokens [t0, t0 + n), logical
 * layout [n][d].  Element (t, j) has counter (g*Lmax + t)*d + j.  If qhat is
 * non-NULL, token 0 gets +6*qhat and heavy tokens +4*qhat (keys only). */
void skvg_host_kv_group(uint64_t seed, uint32_t layer, uint64_t g, uint64_t Lmax, uint64_t t0,
                        uint64_t n, int d, const double* qhat, uint16_t* K, uint16_t* V) {
  uint64_t kk = skvg_key(seed, SKVG_S_K, layer);
  uint64_t kv = skvg_key(seed, SKVG_S_V, layer);
  uint64_t kh = skvg_key(seed, SKVG_S_HEAVY, layer);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)n; ++i) {
    uint64_t t = t0 + (uint64_t)i;
    double coef = 0.0;
    if (qhat) coef = (t == 0) ? 6.0 : (skvg_is_heavy(kh, g, Lmax, t) ? 4.0 : 0.0);
    for (int j = 0; j < d; ++j) {
      uint64_t c = (g * Lmax + t) * (uint64_t)d + (uint64_t)j;
      uint16_t k = skvg_normal_bf16(kk, c);
      if (coef != 0.0) k = skvg_shift_bf16(k, coef, qhat[j]);
      if (K) K[(uint64_t)i * d + j] = k;
      if (V) V[(uint64_t)i * d + j] = skvg_normal_bf16(kv, c);
    }
  }
}

/* Cluster sizes -> offsets for one group: slot i in [0, L) draws a component;
 * counting the draws and taking the exclusive prefix sum gives contiguous
 * clusters [off[c], off[c+1]). off has C+1 entries, C = 2^c_log2. */
void skvg_host_mixture_offsets(uint64_t seed, uint32_t layer, uint64_t g, uint64_t Lmax,
                               uint64_t L, uint32_t c_log2, int32_t* off) {
  uint64_t ka = skvg_key(seed, SKVG_S_ASSIGN, layer);
  uint32_t C = 1u << c_log2;
  memset(off, 0, sizeof(int32_t) * (C + 1));
  for (uint64_t i = 0; i < L; ++i) off[skvg_component(ka, g, Lmax, i, c_log2) + 1] += 1;
  for (uint32_t c = 0; c < C; ++c) off[c + 1] += off[c];
}

/* Mixture keys of group g in sorted (cluster-contiguous) order, [L][d], and the
 * bf16 centroids [C][d] (fp64 mean of the member keys, ascending token order;
 * an empty cluster's centroid is its center). off from skvg_host_mixture_offsets. */
void skvg_host_mixture_group(uint64_t seed, uint32_t layer, uint64_t g, uint64_t Lmax, uint64_t L,
                             int d, uint32_t c_log2, const int32_t* off, uint16_t* K,
                             uint16_t* centroids) {
  uint64_t kc = skvg_key(seed, SKVG_S_CENTER, layer);
  uint64_t kk = skvg_key(seed, SKVG_S_K, layer);
  uint32_t C = 1u << c_log2;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t c = 0; c < (int64_t)C; ++c) {
    for (int j = 0; j < d; ++j) {
      uint16_t center = skvg_normal_bf16(kc, (g * C + (uint64_t)c) * (uint64_t)d + (uint64_t)j);
      double sum = 0.0;
      for (int32_t t = off[c]; t < off[c + 1]; ++t) {
        float nz = skvg_normal(kk, (g * Lmax + (uint64_t)t) * (uint64_t)d + (uint64_t)j);
        uint16_t k = skvg_mixture_key(center, nz);
        if (K) K[(uint64_t)t * d + j] = k;
        sum = SKVG_DADD(sum, skvg_bf16_to_f64(k));
      }
      int32_t sz = off[c + 1] - off[c];
      if (centroids)
        centroids[(uint64_t)c * d + j] =
            sz > 0 ? skvg_f64_to_bf16(SKVG_DDIV(sum, (double)sz)) : center;
    }
  }
  (void)L;
}

/* Seeded Fisher-Yates permutation of [0, n) (uniform index by multiply-shift). */
void skvg_host_perm(uint64_t seed, uint32_t stream, uint32_t layer, int32_t n, int32_t* out) {
  uint64_t key = skvg_key(seed, stream, layer);
  for (int32_t i = 0; i < n; ++i) out[i] = i;
  for (int32_t i = n - 1; i > 0; --i) {
    uint64_t h = skvg_hash(key, (uint64_t)i);
    int32_t j = (int32_t)(((h >> 32) * (uint64_t)(i + 1)) >> 32);
    int32_t tmp = out[i];
    out[i] = out[j];
    out[j] = tmp;
  }
}

int skvg_host_route_bit(uint64_t seed, uint32_t layer) {
  return skvg_route_bit(skvg_key(seed, SKVG_S_ROUTE, 0), layer);
}

int skvg_host_is_heavy(uint64_t seed, uint32_t layer, uint64_t g, uint64_t Lmax, uint64_t t) {
  return skvg_is_heavy(skvg_key(seed, SKVG_S_HEAVY, layer), g, Lmax, t);
}

uint16_t skvg_host_f64_to_bf16(double x) { return skvg_f64_to_bf16(x); }
uint16_t skvg_host_f32_to_bf16(float x) { return skvg_f32_to_bf16(x); }

/* Block summaries of one KV group: out[j][:] = bf16( fp64 mean of the keys
 * K[t][:] of block j, t in [j*bs, min((j+1)*bs, L)) ), ascending t. */
void skvg_host_block_means(const uint16_t* K, uint64_t L, int d, int bs, uint16_t* out) {
  uint64_t nb = (L + (uint64_t)bs - 1) / (uint64_t)bs;
  for (uint64_t blk = 0; blk < nb; ++blk) {
    uint64_t t0 = blk * (uint64_t)bs, t1 = t0 + (uint64_t)bs < L ? t0 + (uint64_t)bs : L;
    for (int j = 0; j < d; ++j) {
      double sum = 0.0;
      for (uint64_t t = t0; t < t1; ++t) sum = SKVG_DADD(sum, skvg_bf16_to_f64(K[t * (uint64_t)d + j]));
      out[blk * (uint64_t)d + j] = skvg_f64_to_bf16(SKVG_DDIV(sum, (double)(t1 - t0)));
    }
  }
}
