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
  int n_splits;
  float qscale;  // softmax scale * log2(e): scores are kept in base-2 units
  float tau, phi;
  int patience;
  float* out;
  float* lse;
  int* blocks_consumed;
  uint32_t* status;
  float* ws_o;    // [n_splits][B*Hq][128] when n_splits > 1
  float* ws_lse;  // [n_splits][B*Hq]
};

// Host-side launchers (decode.cu / merge.cu / select.cu).
int launch_decode(const DecodeParams& p, int G, bool art, void* stream);
int launch_merge(const float* o_parts, const float* lse_parts, int S, int N, int d, float* out,
                 float* lse, void* stream);
int launch_select(const uint16_t* q, const uint16_t* cent, const int* off, int B, int Hq, int Hkv,
                  int C, int k, int* ids, int* ss, int* se, void* stream);
int num_sms();

}  // namespace skv
