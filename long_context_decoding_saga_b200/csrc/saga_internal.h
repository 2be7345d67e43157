// saga_internal.h - parameter blocks shared by the host launchers and the
// kernels, and the workspace layout.  Not part of the public ABI.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "saga.h"

namespace saga {

constexpr int kTile = 128;       // tokens per pipeline tile (UMMA M)
constexpr int kUnit = 32;        // split boundaries fall on multiples of 32 tokens
constexpr int kEpiThreads = 128; // epilogue warps: one thread per token of a tile
constexpr int kMaxG = 64;        // query heads per key head
constexpr int kMaxNvh = 32;      // value heads per key-head group
constexpr int kMaxCtasPerSm = 4; // bound used to size the split partials
constexpr int kSelectThreads = 1024;
constexpr int kSelectCap = 16384; // radix-select candidates kept in shared memory

// Token range [start, end) of split s out of S over a row of L tokens.
__host__ __device__ inline void split_range(int L, int S, int s, int* start, int* end) {
  const long long U = (L + kUnit - 1) / kUnit;
  const long long a = (s * U) / S, b = ((s + 1) * U) / S;
  long long st = a * kUnit, en = b * kUnit;
  if (en > L) en = L;
  if (st > L) st = L;
  *start = (int)st;
  *end = (int)en;
}

// Byte offsets of the workspace regions (each 256-byte aligned).
struct WsLayout {
  size_t status;    // unsigned status word
  size_t part_o;    // float [B*h_q, S_cap, d]
  size_t part_m;    // float [B*h_q, S_cap]
  size_t part_l;    // float [B*h_q, S_cap]
  size_t part_cnt;  // int   [B*h_q, S_cap]
  size_t scores;    // float [B*h_q, ld_scores]
  size_t hist;      // uint32 [B*h_q, 256]
  size_t idx;       // int   [B*h_q, l_cap]
  size_t total;
  int s_cap;
  long long ld_scores;
};

struct SplitParams {
  const uint16_t* q;        // bf16 [B, h_q, d]
  const uint16_t* v_cache;  // bf16 [B, h_v, l_cap, d]
  const float* tau;         // [B, h_q]
  const float* scores_in;   // from-scores mode: [B*h_q, ld_scores]
  float* scores_out;        // dump mode
  uint32_t* hist_out;       // dump mode: [B*h_q, 256]
  float* part_o;
  float* part_m;
  float* part_l;
  int* part_cnt;
  int* idxbuf;              // nullable
  unsigned* status;
  const int* seq_len_dev;   // nullable
  long long ld_scores;
  int seq_len;
  int batch, h_q, h_k, h_v, l_cap;
  int nsplit;    // splits per (batch, key head)
  int s_cap;     // partials stride
  int G;         // h_q / h_k
  int nvh;       // value heads per key-head group
  int hpv;       // query heads of the group per value head
  float scale;   // fp32(1/sqrt(d))
  int want_counts;
};

struct CombineParams {
  const float* part_o;
  const float* part_m;
  const float* part_l;
  const int* part_cnt;
  const int* idxbuf;
  void* out;
  int* sel_count;
  int* sel_idx;
  unsigned* status;
  const int* seq_len_dev;
  int seq_len;
  int rows;      // B * h_q
  int nsplit;
  int s_cap;
  int l_cap;
  int out_bf16;
};

struct SelectParams {
  const float* scores;
  long long ld;
  const uint32_t* hist;  // nullable: precomputed top-byte histogram [rows, 256]
  float* tau;
  unsigned* status;
  const int* seq_len_dev;  // nullable: row length from the device
  int row_len;
  int l_cap;               // clamp bound for a device length
  int n_top;
};

struct AppendParams {
  uint16_t* k_cache;
  uint16_t* v_cache;
  const uint16_t* k_new;
  const uint16_t* v_new;
  const int* seq_len_dev;
  unsigned* status;
  int pos;
  int batch, h_k, h_v, d, l_cap;
};

// Reads the effective sequence length on the device, clamped to [1, l_cap].
__device__ inline int device_seq_len(const int* dev, int host_len, int l_cap, unsigned* status) {
  if (dev == nullptr) return host_len;
  int L = *reinterpret_cast<const volatile int*>(dev);
  if (L < 1 || L > l_cap) {
    if (status) atomicOr(status, SAGA_STATUS_LEN_CLAMPED);
    L = L < 1 ? 1 : l_cap;
  }
  return L;
}

}  // namespace saga
