// api.cu -- the C ABI of libsparsekv.so: host-side validation, the launch
// plan (split count, workspace carve-up) and the launches.  No exception or
// exit crosses this boundary; every path returns an skv_status.
#include <math.h>
#include <algorithm>
#include <atomic>
#include <stdint.h>

#include <cuda_runtime.h>

#include "../../include/sparsekv.h"
#include "common.cuh"
#include "decode.cuh"

#ifndef SKV_ART_AHEAD
#define SKV_ART_AHEAD 0
#endif

namespace skv {
namespace {

struct Plan {
  int G = 0;
  bool chunk = false;
  int mode = TRAV_NATURAL;
  bool art = false;
  int sched = SCHED_PERSISTENT;
  int n_ctas = 0;
  int splits = 1;
  int nw = 0;
  size_t hdr_bytes = 0;   // plain: header; ART: zeroed control words
  size_t lb_bytes = 0;    // ART look-back records
  size_t scratch_bytes = 0;  // ART per-CTA scratch
  size_t ws_bytes = 0;
  int art_chunk = 0, art_maxc = 0, art_ahead = 0;
};

// Pending test hook of skv_test_withhold_tile: (cta << 32) | entry, 0 = none.
std::atomic<unsigned long long> g_withhold{0};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

// Split count for traversals of up to n_tiles tiles per group: minimise
// (waves x tiles per CTA) plus a per-wave fill cost, given the resident CTAs per SM.
int choose_splits(long long groups, long long n_tiles, int ctas_per_sm, int max_splits) {
  if (n_tiles <= 1 || groups <= 0) return 1;
  const int sms = num_sms() * ctas_per_sm;
  const int s_max = (int)std::max<long long>(1, std::min<long long>(max_splits, n_tiles / 4));
  int best = 1;
  long long best_cost = -1;
  for (int s = 1; s <= s_max; ++s) {
    const long long waves = (groups * s + sms - 1) / sms;
    const long long cost = waves * (cdiv(n_tiles, s) + 2);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

skv_status make_plan(const skv_decode_args* a, Plan* pl) {
  if (!a) return SKV_EINVAL;
  if (!a->q || !a->k_pool || !a->v_pool || !a->block_table || !a->seq_lens || !a->out || !a->lse)
    return SKV_EINVAL;
  if (a->batch < 1 || a->q_tokens < 1 || a->q_heads < 1 || a->kv_heads < 1) return SKV_EINVAL;
  if (a->q_heads % a->kv_heads != 0) return SKV_EINVAL;
  if (a->max_seq_len < 0 || a->num_pages < 1 || a->max_blocks < 0) return SKV_EINVAL;
  if (a->head_dim != kHeadDim || a->block_size != kBlock) return SKV_EUNSUPPORTED;
  if ((long long)a->max_blocks * kBlock < (long long)a->max_seq_len) return SKV_EINVAL;
  if (!aligned16(a->q) || !aligned16(a->out) || !aligned16(a->k_pool) || !aligned16(a->v_pool))
    return SKV_EINVAL;
  if (!isfinite(a->scale)) return SKV_EINVAL;
  const int G = a->q_heads / a->kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SKV_EUNSUPPORTED;
  if (a->kv_shards < 0) return SKV_EINVAL;

  const bool has_order = a->order != nullptr;
  const bool has_seg = a->seg_start != nullptr || a->seg_end != nullptr;
  const bool has_win = a->window.sink_tokens != 0 || a->window.recent_tokens != 0;
  const bool has_range = a->kv_end > 0 || a->kv_begin != 0;
  if ((int)has_order + (int)has_seg + (int)has_win + (int)has_range > 1) return SKV_EUNSUPPORTED;
  if (has_order && a->order_len < 0) return SKV_EINVAL;
  if (has_seg && (!a->seg_start || !a->seg_end || a->n_seg < 0)) return SKV_EINVAL;
  if (has_win && (a->window.sink_tokens < 0 || a->window.recent_tokens < 0)) return SKV_EINVAL;
  if (has_range && (a->kv_begin < 0 || a->kv_end < a->kv_begin)) return SKV_EINVAL;
  if (a->art.enable) {
    if (!(a->art.tau >= 0.f) || !(a->art.phi >= 0.f) || a->art.patience < 1) return SKV_EINVAL;
    if (has_seg || has_win || has_range) return SKV_EUNSUPPORTED;
  }
  if (a->q_tokens > 1) {  // query chunk on the tensor cores
    if (a->art.enable || has_order || has_seg || has_win) return SKV_EUNSUPPORTED;
    pl->G = G;
    pl->chunk = true;
    pl->art = false;
    pl->mode = TRAV_NATURAL;
    pl->ws_bytes = 0;
    return SKV_OK;
  }
  if (a->kv_shards > 1) return SKV_EUNSUPPORTED;  // decode: one result (use kv ranges)

  pl->G = G;
  pl->art = a->art.enable != 0;
  pl->mode = has_order ? TRAV_ORDER : has_seg ? TRAV_SEGMENTS : has_win ? TRAV_WINDOW : TRAV_NATURAL;
  pl->splits = 1;
  pl->n_ctas = 0;
  pl->hdr_bytes = 0;
  pl->ws_bytes = 0;
  const long long groups = (long long)a->batch * a->kv_heads;
  if (pl->art) {
    // (chunk, group) items; one record per (group, chunk, head)
    DecodeParams probe{};
    probe.mode = pl->mode;
    probe.order_len = a->order_len;
    pl->sched = SCHED_ART;
    pl->nw = 1;
    pl->n_ctas = num_sms() * art_ctas_per_sm(G);
    const long long positions = art_positions(probe, a->max_seq_len);
    pl->art_chunk = art_chunk_blocks(G, pl->n_ctas, groups, positions);
    pl->art_maxc = (int)cdiv(positions, pl->art_chunk);
    // speculation gate (SKV_ART_AHEAD > 0: that many times the chunks in flight
    // per group at the start), off by default
    pl->art_ahead = SKV_ART_AHEAD > 0
                        ? (int)(SKV_ART_AHEAD * std::max<long long>(1, cdiv(pl->n_ctas, groups)))
                        : (1 << 30);
    const long long items = groups * pl->art_maxc;
    if (items >= (1ll << 30) || pl->art_maxc > 32768) return SKV_EUNSUPPORTED;
    pl->hdr_bytes = (size_t)cdiv(art_ctl_words(groups, pl->art_maxc, G) * 4, 256) * 256;
    pl->lb_bytes = (size_t)cdiv(items * G * kLbFloats * 4, 256) * 256;
    pl->scratch_bytes = (size_t)pl->n_ctas * art_scratch_bytes_per_cta(G, pl->art_chunk);
    pl->ws_bytes = pl->hdr_bytes + pl->lb_bytes + pl->scratch_bytes +
                   (size_t)items * G * kRecFloats * sizeof(float);
    return SKV_OK;
  }
  pl->nw = decode_consumer_warps(G);
  DecodeParams probe{};
  probe.mode = pl->mode;
  probe.range_begin = a->kv_begin;
  probe.range_end = a->kv_end;
  probe.sink = a->window.sink_tokens;
  probe.recent = a->window.recent_tokens;
  probe.order_len = a->order_len;
  const long long t_est =
      pl->mode == TRAV_SEGMENTS ? 0 : groups * group_tiles(probe, a->max_seq_len);
  if (t_est >= (1ll << 31)) return SKV_EUNSUPPORTED;
  // Small walks (a few tiles per resident CTA) are latency-bound: there the
  // split schedule, which merges inside the kernel, saves the second launch.
  const long long small = (long long)num_sms() * decode_ctas_per_sm(G) * 8;
  if (pl->mode != TRAV_SEGMENTS && a->batch <= kMaxPersistentBatch && t_est > small) {
    pl->sched = SCHED_PERSISTENT;
    const long long max_ctas = (long long)num_sms() * decode_ctas_per_sm(G);
    pl->n_ctas = (int)std::max<long long>(1, std::min<long long>(max_ctas, cdiv(t_est, 4)));
    const long long slots = pl->n_ctas + groups;
    pl->hdr_bytes = (size_t)cdiv((a->batch + 2) * 4ll, 256) * 256;
    pl->ws_bytes = pl->hdr_bytes + (size_t)slots * pl->nw * G * kRecFloats * sizeof(float);
  } else {
    // one cluster of `splits` CTAs per group, merged in distributed shared
    // memory: no workspace
    pl->sched = SCHED_SPLIT;
    pl->splits = choose_splits(groups, pl->mode == TRAV_SEGMENTS ? a->n_seg : cdiv(a->max_seq_len, kBlock),
                               decode_ctas_per_sm(G), kMaxClusterSplits);
    pl->ws_bytes = 0;
  }
  return SKV_OK;
}

}  // namespace
}  // namespace skv

using namespace skv;

extern "C" {

size_t skv_decode_workspace_size(const skv_decode_args* args) {
  Plan pl;
  if (make_plan(args, &pl) != SKV_OK) return 0;
  return pl.ws_bytes;
}

int skv_decode_launches(const skv_decode_args* args) {
  Plan pl;
  if (make_plan(args, &pl) != SKV_OK) return 0;
  return (pl.chunk || (!pl.art && pl.sched == SCHED_SPLIT)) ? 1 : 2;
}

skv_status skv_decode_plan_info(const skv_decode_args* args, skv_decode_plan* plan) {
  if (!plan) return SKV_EINVAL;
  *plan = skv_decode_plan{};
  Plan pl;
  const skv_status st = make_plan(args, &pl);
  if (st != SKV_OK) return st;
  plan->launches = (pl.chunk || (!pl.art && pl.sched == SCHED_SPLIT)) ? 1 : 2;
  plan->workspace_bytes = pl.ws_bytes;
  if (pl.chunk) {
    plan->schedule = SKV_SCHED_CHUNK;
  } else if (pl.art) {
    plan->schedule = SKV_SCHED_ART;
    plan->ctas = pl.n_ctas;
    plan->art_chunk_blocks = pl.art_chunk;
    plan->art_chunks = pl.art_maxc;
  } else if (pl.sched == SCHED_PERSISTENT) {
    plan->schedule = SKV_SCHED_PERSISTENT;
    plan->ctas = pl.n_ctas;
  } else {
    plan->schedule = SKV_SCHED_CLUSTER;
    plan->splits = pl.splits;
    plan->ctas = pl.splits * args->kv_heads * args->batch;
  }
  return SKV_OK;
}

skv_status attn_decode(const skv_decode_args* a, skv_stream_t stream) {
  Plan pl;
  const skv_status st = make_plan(a, &pl);
  if (st != SKV_OK) return st;
  if (pl.ws_bytes > 0 &&
      (!a->workspace || a->workspace_bytes < pl.ws_bytes || !aligned16(a->workspace)))
    return SKV_EWORKSPACE;

  DecodeParams p{};
  p.q = static_cast<const uint16_t*>(a->q);
  p.k_pool = static_cast<const uint16_t*>(a->k_pool);
  p.v_pool = static_cast<const uint16_t*>(a->v_pool);
  p.block_table = a->block_table;
  p.seq_lens = a->seq_lens;
  p.order = a->order;
  p.order_len = a->order_len;
  p.seg_start = a->seg_start;
  p.seg_end = a->seg_end;
  p.n_seg = a->n_seg;
  p.B = a->batch;
  p.Hq = a->q_heads;
  p.Hkv = a->kv_heads;
  p.max_blocks = a->max_blocks;
  p.num_pages = a->num_pages;
  p.max_seq_len = a->max_seq_len;
  p.range_begin = a->kv_begin;
  p.range_end = a->kv_end;
  p.sink = a->window.sink_tokens;
  p.recent = a->window.recent_tokens;
  p.mode = pl.mode;
  p.sched = pl.sched;
  p.n_ctas = pl.n_ctas;
  p.n_splits = pl.splits;
  p.qscale = a->scale * 1.4426950408889634f;
  p.tau = a->art.tau;
  p.phi = a->art.phi;
  p.patience = a->art.patience;
  p.out = a->out;
  p.lse = a->lse;
  p.blocks_consumed = a->blocks_consumed;
  p.status = a->status_word;
  p.rec_nw = pl.nw;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (pl.chunk) {
    if (launch_chunk(p, a->q_tokens, a->causal, a->kv_shards, s) != 0) return SKV_ECUDA;
    return SKV_OK;
  }
  char* ws = static_cast<char*>(a->workspace);
  if (pl.art) {
    p.art_chunk = pl.art_chunk;
    p.art_maxc = pl.art_maxc;
    p.art_ahead = pl.art_ahead;
    p.art_ctl = reinterpret_cast<int*>(ws);
    p.art_lb = reinterpret_cast<float*>(ws + pl.hdr_bytes);
    p.art_scratch = reinterpret_cast<float*>(ws + pl.hdr_bytes + pl.lb_bytes);
    p.ws_rec = reinterpret_cast<float*>(ws + pl.hdr_bytes + pl.lb_bytes + pl.scratch_bytes);
    if (cudaMemsetAsync(ws, 0, pl.hdr_bytes, s) != cudaSuccess) return SKV_ECUDA;
    if (launch_art(p, pl.G, s) != 0) return SKV_ECUDA;
  } else {
    p.ws_hdr = reinterpret_cast<int*>(ws);
    p.ws_rec = reinterpret_cast<float*>(ws + pl.hdr_bytes);
    const unsigned long long wh = g_withhold.exchange(0ull);
    if (wh != 0ull) {
      p.withhold_cta = (int)(wh >> 32);
      p.withhold_entry = (int)(wh & 0xFFFFFFFFull);
    }
    if (launch_decode(p, pl.G, s) != 0) return SKV_ECUDA;
    if (pl.sched == SCHED_SPLIT) return SKV_OK;  // merged inside the kernel
  }
  if (launch_merge_records(p, pl.G, s) != 0) return SKV_ECUDA;
  return SKV_OK;
}

skv_status attn_select_centroids(const void* q, const void* centroids, const int32_t* cluster_off,
                                 int batch, int q_heads, int kv_heads, int head_dim, int n_clusters,
                                 int topk, int32_t* sel_ids, int32_t* seg_start, int32_t* seg_end,
                                 skv_stream_t stream) {
  if (!q || !centroids || !cluster_off || !sel_ids || !seg_start || !seg_end) return SKV_EINVAL;
  if (batch < 1 || q_heads < 1 || kv_heads < 1 || q_heads % kv_heads != 0) return SKV_EINVAL;
  if (n_clusters < 1 || topk < 1 || topk > n_clusters) return SKV_EINVAL;
  if (head_dim != kHeadDim || n_clusters > 4096) return SKV_EUNSUPPORTED;
  if (!aligned16(q) || !aligned16(centroids)) return SKV_EINVAL;
  if (launch_select(static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(centroids),
                    cluster_off, batch, q_heads, kv_heads, n_clusters, topk, 0, sel_ids, seg_start,
                    seg_end, reinterpret_cast<cudaStream_t>(stream)) != 0)
    return SKV_ECUDA;
  return SKV_OK;
}

skv_status attn_select_centroids_shared(const void* q, const void* centroids,
                                        const int32_t* cluster_off, int batch, int q_heads,
                                        int kv_heads, int head_dim, int n_clusters, int topk,
                                        int32_t* sel_ids, int32_t* seg_start, int32_t* seg_end,
                                        skv_stream_t stream) {
  if (!q || !centroids || !cluster_off || !sel_ids || !seg_start || !seg_end) return SKV_EINVAL;
  if (batch < 1 || q_heads < 1 || kv_heads < 1 || q_heads % kv_heads != 0) return SKV_EINVAL;
  if (n_clusters < 1 || topk < 1 || topk > n_clusters) return SKV_EINVAL;
  if (head_dim != kHeadDim || n_clusters > 4096) return SKV_EUNSUPPORTED;
  if (batch > 65535 * 8) return SKV_EUNSUPPORTED;
  if (!aligned16(q) || !aligned16(centroids)) return SKV_EINVAL;
  if (launch_select(static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(centroids),
                    cluster_off, batch, q_heads, kv_heads, n_clusters, topk, 1, sel_ids, seg_start,
                    seg_end, reinterpret_cast<cudaStream_t>(stream)) != 0)
    return SKV_ECUDA;
  return SKV_OK;
}

skv_status attn_merge_lse(const float* o_parts, const float* lse_parts, int n_parts, int n_rows,
                          int head_dim, float* out, float* lse, skv_stream_t stream) {
  if (!o_parts || !lse_parts || !out || !lse) return SKV_EINVAL;
  if (n_parts < 1 || n_rows < 0 || head_dim < 4 || head_dim % 4 != 0 || head_dim > 512)
    return SKV_EINVAL;
  if (!aligned16(o_parts) || !aligned16(out)) return SKV_EINVAL;
  if (launch_merge(o_parts, lse_parts, n_parts, n_rows, head_dim, out, lse,
                   reinterpret_cast<cudaStream_t>(stream)) != 0)
    return SKV_ECUDA;
  return SKV_OK;
}

skv_status attn_forecast(const void* x, const void* w, int batch, int kv_heads, int head_dim, void* f,
                         skv_stream_t stream) {
  if (!x || !w || !f) return SKV_EINVAL;
  if (batch < 1 || kv_heads < 1 || batch > 65535 || kv_heads > 65535) return SKV_EINVAL;
  if (head_dim != kHeadDim) return SKV_EUNSUPPORTED;
  if (launch_forecast(static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(w), batch, kv_heads,
                      static_cast<uint16_t*>(f), reinterpret_cast<cudaStream_t>(stream)) != 0)
    return SKV_ECUDA;
  return SKV_OK;
}

skv_status skv_host_device_pointer(const void* host, void** dev) {
  if (!host || !dev) return SKV_EINVAL;
  void* p = nullptr;
  if (cudaHostGetDevicePointer(&p, const_cast<void*>(host), 0) != cudaSuccess || !p) {
    cudaGetLastError();  // the failed query's error is not sticky: clear it
    return SKV_EINVAL;
  }
  *dev = p;
  return SKV_OK;
}

skv_status attn_prefetch_blocks(const void* k_host, const void* v_host, const int32_t* block_table,
                                const int32_t* seq_lens, const int32_t* block_ids, int batch,
                                int kv_heads, int head_dim, int topk, int max_blocks, int num_pages,
                                int max_seq_len, void* k_cache, void* v_cache, int32_t* seg_start,
                                int32_t* seg_end, uint32_t* status_word, int n_ctas,
                                skv_stream_t stream) {
  if (!k_host || !v_host || !block_table || !seq_lens || !block_ids || !k_cache || !v_cache ||
      !seg_start || !seg_end)
    return SKV_EINVAL;
  if (batch < 1 || kv_heads < 1 || topk < 1 || max_blocks < 0 || num_pages < 1 || max_seq_len < 0 ||
      n_ctas < 1 || n_ctas > 65535)
    return SKV_EINVAL;
  if (head_dim != kHeadDim) return SKV_EUNSUPPORTED;
  if ((long long)max_blocks * kBlock < (long long)max_seq_len) return SKV_EINVAL;
  if (!aligned16(k_host) || !aligned16(v_host) || !aligned16(k_cache) || !aligned16(v_cache))
    return SKV_EINVAL;
  if (launch_gather(k_host, v_host, block_table, seq_lens, block_ids, batch, kv_heads, topk, max_blocks,
                    num_pages, max_seq_len, k_cache, v_cache, seg_start, seg_end, status_word, n_ctas,
                    reinterpret_cast<cudaStream_t>(stream)) != 0)
    return SKV_ECUDA;
  return SKV_OK;
}

skv_status skv_test_withhold_tile(int cta, int entry) {
  if (cta < 0) {  // clear a pending hook
    g_withhold.store(0ull);
    return SKV_OK;
  }
  if (entry < 0 || entry > 0x7FFFFFFE) return SKV_EINVAL;
  g_withhold.store(((unsigned long long)(unsigned)cta << 32) | (unsigned long long)(entry + 1));
  return SKV_OK;
}

skv_status skv_status_of_word(uint32_t word) {
  if (word & SKV_DEV_TIMEOUT) return SKV_ETIMEOUT;
  if (word & (SKV_DEV_BAD_PAGE | SKV_DEV_BAD_SEQLEN | SKV_DEV_BAD_ORDER | SKV_DEV_BAD_SEGMENT))
    return SKV_EINVAL;
  return SKV_OK;
}

const char* skv_strerror(skv_status s) {
  switch (s) {
    case SKV_OK: return "ok";
    case SKV_EINVAL: return "invalid argument";
    case SKV_EUNSUPPORTED: return "unsupported shape or option combination";
    case SKV_ECUDA: return "CUDA runtime error";
    case SKV_ETIMEOUT: return "device wait timed out";
    case SKV_EWORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

}  // extern "C"
