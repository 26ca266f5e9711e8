// decode.cuh -- launch-plan types shared by the C-ABI layer and the kernels.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace skv {

enum TravMode : int {
  TRAV_NATURAL = 0,   // blocks 0..nb-1 (or a [kv_begin, kv_end) token range)
  TRAV_ORDER = 1,     // caller's list of logical blocks
  TRAV_WINDOW = 2,    // sink + recent window
  TRAV_SEGMENTS = 3,  // caller's token segments
};

enum Schedule : int {
  SCHED_PERSISTENT = 0,  // one CTA per SM walks an even share of all tiles of all groups
  SCHED_SPLIT = 1,       // grid (splits, kv_heads, batch), a cluster per group, merged in-kernel
  SCHED_ART = 2,         // persistent CTAs take (chunk, group) items (art.cu)
};

constexpr int kMaxPersistentBatch = 1024;  // batch prefix kept in shared memory
constexpr int kMaxClusterSplits = 16;      // split schedule: CTAs per cluster (one group)
constexpr int kRecFloats = 132;            // partial record: O[128], m (base 2), l, tiles, pad
constexpr int kLbFloats = 12;              // ART look-back record per head: m, l, O[0:8], run, state

struct DecodeParams {
  const uint16_t* q;
  const uint16_t* k_pool;
  const uint16_t* v_pool;
  const int* block_table;
  const int* seq_lens;
  const int* order;
  int order_len;
  const int* seg_start;
  const int* seg_end;
  int n_seg;
  int B, Hq, Hkv, max_blocks, num_pages, max_seq_len;
  int range_begin, range_end;  // token range (range_end > 0 => active)
  int sink, recent;
  int mode;
  int sched;
  int n_ctas;    // SCHED_PERSISTENT: grid size
  int n_splits;  // SCHED_SPLIT: pieces per group
  float qscale;  // softmax scale * log2(e): scores are kept in base-2 units
  float tau, phi;
  int patience;
  float* out;
  float* lse;
  int* blocks_consumed;
  uint32_t* status;
  // Non-ART workspace: header (total tiles, batch prefix) and per-warp partial
  // records [slots][rec_nw][G][kRecFloats], merged by launch_merge_records.
  int* ws_hdr;
  float* ws_rec;
  int rec_nw;
  // ART (SCHED_ART): chunk length in blocks, chunks per group (the longest
  // sequence's), control words zeroed before every launch (item counter, stop
  // chunk per group, ready flag per chunk, blocks consumed and stop chunk per
  // head) and the
  // look-back records [group][chunk][G][kLbFloats]; ws_rec holds one record
  // per (group, chunk, head) (rec_nw = 1).
  int art_chunk;
  int art_maxc;
  int art_ahead;  // a group's chunk c starts once chunk c - art_ahead - 1 is decided
  int* art_ctl;
  float* art_lb;
  float* art_scratch;  // per-CTA probe slots and state area (stays in L2)
  // Test hook (skv_test_withhold_tile): when withhold_entry > 0, the producer of
  // CTA withhold_cta (linear block index) stops before ring entry
  // withhold_entry - 1, so that the consumers' bounded wait for it expires.
  int withhold_cta, withhold_entry;
};

// ART traversal positions of a sequence of L tokens: block 0, then the
// caller's list (with block 0 skipped) or the other blocks most recent first.
__host__ __device__ inline int art_positions(const DecodeParams& p, int L) {
  const int nb = (L + 63) / 64;
  if (nb == 0) return 0;
  return p.mode == TRAV_ORDER ? 1 + p.order_len : nb;
}

// Control words of the ART schedule: counter (4), stop chunk per group, ready
// flag per chunk, blocks consumed and stop chunk per head.
inline long long art_ctl_words(long long groups, long long maxc, int G) {
  return 4 + groups + groups * maxc + 2 * groups * G;
}

// Tiles of one KV group for the index-based traversals (natural / range /
// window / order), given the sequence length L.
__host__ __device__ inline int group_tiles(const DecodeParams& p, int L) {
  const int nb = (L + 63) / 64;
  switch (p.mode) {
    case TRAV_NATURAL: {
      int ra = 0, re = L;
      if (p.range_end > 0) {
        ra = p.range_begin > 0 ? p.range_begin : 0;
        re = p.range_end < L ? p.range_end : L;
      }
      return (re > ra) ? (re + 63) / 64 - ra / 64 : 0;
    }
    case TRAV_WINDOW: {
      const int A = p.sink < L ? p.sink : L;
      const int Rs = (L - p.recent > A) ? L - p.recent : A;
      return (A + 63) / 64 + ((L > Rs) ? nb - Rs / 64 : 0);
    }
    case TRAV_ORDER: return p.order_len;
    default: return 0;
  }
}

// Host-side launchers (decode.cu / merge.cu / select.cu).
int launch_decode(const DecodeParams& p, int G, void* stream);
int decode_consumer_warps(int G);
int decode_ctas_per_sm(int G);
int launch_art(const DecodeParams& p, int G, void* stream);
int art_chunk_blocks(int G, long long n_ctas, long long groups, long long positions);
int art_ctas_per_sm(int G);
size_t art_scratch_bytes_per_cta(int G, int CB);
int launch_merge(const float* o_parts, const float* lse_parts, int S, int N, int d, float* out,
                 float* lse, void* stream);
int launch_merge_records(const DecodeParams& p, int G, void* stream);
int launch_chunk(const DecodeParams& p, int Tq, int causal, int n_shards, void* stream);
int launch_select(const uint16_t* q, const uint16_t* cent, const int* off, int B, int Hq, int Hkv,
                  int C, int k, int shared, int* ids, int* ss, int* se, void* stream);
int select_cluster_size(int B);
int launch_forecast(const uint16_t* x, const uint16_t* w, int B, int Hkv, uint16_t* f, void* stream);
int launch_gather(const void* k_host, const void* v_host, const int* block_table, const int* seq_lens,
                  const int* ids, int B, int Hkv, int k, int max_blocks, int num_pages, int max_seq_len,
                  void* k_cache, void* v_cache, int* seg_start, int* seg_end, uint32_t* status,
                  int n_ctas, void* stream);
int num_sms();

}  // namespace skv
