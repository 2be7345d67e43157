// saga_internal.h - parameter blocks shared by the host launchers and the
// kernels, and the workspace layout.  Not part of the public ABI.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "saga.h"

namespace saga {

// Split-kernel modes: attend with every token kept (N covers every length),
// attend with the Atop-N threshold, or dump scores for a refresh.
constexpr int kSplitDense = 0, kSplitSparse = 1, kSplitDump = 2;
constexpr int kTile = 128;       // tokens per pipeline tile (UMMA M)
constexpr int kUnit = 32;        // split boundaries fall on multiples of 32 tokens
constexpr int kEpiThreads = 128; // epilogue warps: one thread per token of a tile
constexpr int kMaxG = 64;        // query heads per key head
constexpr int kMaxNvh = 32;      // value heads per key-head group
constexpr int kMaxCtasPerSm = 4; // bound used to size the split partials
constexpr int kSelectThreads = 1024;
constexpr int kSelectCap = 16384; // radix-select candidates kept in shared memory

// Token range [start, end) of split s out of S.  The boundaries partition P
// tokens (the host's length at launch, fixed for a captured graph) at
// multiples of kUnit; the range is then clamped to the device length L, and
// the last split also takes any tokens in [P, L).
__host__ __device__ inline void split_range(int P, int S, int s, int L, int* start, int* end) {
  const long long U = (P + kUnit - 1) / kUnit;
  const long long a = (s * U) / S, b = ((s + 1) * U) / S;
  long long st = a * kUnit, en = (s == S - 1) ? (long long)L : b * kUnit;
  if (en > L) en = L;
  if (st > L) st = L;
  *start = (int)st;
  *end = (int)en;
}

// Rows split s may cover whatever the device length is: [start, cap_end),
// within the cache capacity (used for prefetching before the length is read).
__host__ __device__ inline void split_cap_range(int P, int S, int s, int l_cap, int* start, int* cap_end) {
  const long long U = (P + kUnit - 1) / kUnit;
  const long long a = (s * U) / S, b = ((s + 1) * U) / S;
  long long st = a * kUnit, en = (s == S - 1) ? (long long)l_cap : b * kUnit;
  if (en > l_cap) en = l_cap;
  if (st > l_cap) st = l_cap;
  *start = (int)st;
  *cap_end = (int)en;
}

// Byte offsets of the workspace regions (each 256-byte aligned).
struct WsLayout {
  size_t status;    // unsigned status word
  size_t part_o;    // float [B*h_q, S_cap, d]
  size_t part_m;    // float [B*h_q, S_cap]
  size_t part_l;    // float [B*h_q, S_cap]
  size_t part_cnt;  // int   [B*h_q, S_cap]
  size_t scores;    // float [B*h_q, ld_scores]
  size_t hist;      // uint32 [B*h_q, 256] top-byte counts of the dumped scores (groups of <= 4 heads)
  size_t idx;       // int   [B*h_q, l_cap]
  size_t total;
  int s_cap;
  long long ld_scores;
};

struct SplitParams {
  const uint16_t* q;        // bf16 [B, h_q, d]
  const uint16_t* k_cache;  // bf16 [B, h_k, l_cap, d] (also behind the tensor maps)
  const uint16_t* v_cache;  // bf16 [B, h_v, l_cap, d]
  uint16_t* k_cache_w;      // fused append: caches written at row L - 1
  uint16_t* v_cache_w;
  const uint16_t* k_new;    // fused append (nullable): bf16 [B, h_k, d]
  const uint16_t* v_new;    //                          bf16 [B, h_v, d]
  const float* tau;         // [B, h_q]
  const float* scores_in;   // from-scores mode: [B*h_q, ld_scores]
  float* scores_out;        // dump mode
  uint32_t* hist_out;       // dump mode, padded groups of <= 4 heads: [B*h_q, 256], else null
  int hist_floor;           // dump mode: count only top-byte bins from two below the stale tau's bin up
  float* part_o;
  float* part_m;
  float* part_l;
  int* part_cnt;
  int* idxbuf;              // nullable
  unsigned* status;
  const int* seq_len_dev;   // nullable
  long long ld_scores;
  int seq_len;   // host length: the length when seq_len_dev is null, and the partition length P
  int batch, h_q, h_k, h_v, l_cap;
  int nsplit;    // splits per (batch, key head)
  int s_cap;     // partials stride
  int G;         // query heads per CTA: h_q / h_k / hsplit
  int hsplit;    // CTAs sharing a key head's query heads (sub-groups of G heads)
  int nvh;       // value heads of a CTA's query heads
  int hpv;       // query heads of the CTA per value head
  float scale;   // fp32(1/sqrt(d))
  int want_counts;
  // failure-detection test hook: when nonzero, the epilogue of an attend
  // launch first waits on a barrier nothing arrives at, for at most this many
  // ns (the pipeline then unwinds and flags SAGA_STATUS_TIMEOUT)
  unsigned test_wait_ns;
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

// The score dump also counts the top byte of the scores near the stale
// threshold (so the select can skip its first pass) only for padded groups of
// at most this many heads: there the counting costs little next to the key
// stream; with 8 or 16 heads per CTA it took half the dump's time or more.
constexpr int kDumpHistMaxNp = 4;

struct SelectParams {
  const float* scores;
  long long ld;
  const uint32_t* hist;  // nullable: top-byte counts [rows, 256] that may hold only the upper bins; a row
                         // whose counted bins hold fewer than n_top scores is counted again
  float* tau;
  unsigned* status;
  const int* seq_len_dev;  // nullable: row length from the device
  int row_len;
  int l_cap;               // clamp bound for a device length
  int n_top;
  int spec;                // tau holds the stale thresholds: the top-digit pass also keeps the keys from the
                           // stale threshold's top-byte bin up, and skips the collection pass when they serve
};

// Decode-step QKV projection (eq. 1) fused with the KV-cache append.
struct QkvParams {
  const uint16_t* x;   // bf16 [B, hidden]
  const uint16_t* w;   // bf16 [(h_q + h_k + h_v) d, hidden]: rows of W_Q, then W_K, then W_V
  uint16_t* q;         // bf16 [B, h_q, d]
  uint16_t* k_cache;   // bf16 [B, h_k, l_cap, d]: row pos written
  uint16_t* v_cache;   // bf16 [B, h_v, l_cap, d]: row pos written
  const int* seq_len_dev;  // nullable: pos = *seq_len_dev - 1 (clamped into [0, l_cap))
  unsigned* status;
  int pos;
  int batch, hidden, n_cols, h_q, h_k, h_v, d, l_cap;
  int splits, kb_total, stages, kbs_max;  // tensor-core path: hidden split (cluster size) and ring depth
};

// Tensor-core QKV projection tiling (shared by the kernel and the workspace sizing).
constexpr int kQkvTileM = 128;    // output columns per tile (MMA M)
constexpr int kQkvTileK = 64;     // hidden elements per k-block: one 128-byte swizzle row
constexpr int kQkvN = 16;         // batch rows of the B operand (MMA N)
constexpr int kQkvMaxStages = 5;  // weight-tile ring depth
constexpr int kQkvMaxKb = 32;     // most k-blocks of x one CTA stages
constexpr int kQkvMaxSplits = 8;  // splits of the hidden dimension: one portable cluster
constexpr int kQkvMaxHidden = kQkvMaxSplits * kQkvMaxKb * kQkvTileK;  // 16384
#ifndef SAGA_QKV_MMA_MIN_BATCH
#define SAGA_QKV_MMA_MIN_BATCH 2
#endif
constexpr int kQkvMmaMinBatch = SAGA_QKV_MMA_MIN_BATCH;  // smallest batch sent to the tensor cores

// Split of the hidden dimension for the tensor-core projection: about one CTA
// per SM over all tiles (at most kQkvMaxSplits, one cluster), each split
// holding at most kQkvMaxKb k-blocks of x (so hidden <= kQkvMaxHidden).
__host__ inline void qkv_mma_plan(int n_cols, int hidden, int sms, int* m_tiles, int* splits, int* kb_total,
                                  int* stages, int* kbs_max) {
  *m_tiles = (n_cols + kQkvTileM - 1) / kQkvTileM;
  *kb_total = (hidden + kQkvTileK - 1) / kQkvTileK;
  int sp = sms / *m_tiles;
  if (sp > kQkvMaxSplits) sp = kQkvMaxSplits;
  if (sp < 1) sp = 1;
  const int need = (*kb_total + kQkvMaxKb - 1) / kQkvMaxKb;
  if (sp < need) sp = need;
  *splits = sp < *kb_total ? sp : *kb_total;
  *kbs_max = (*kb_total + *splits - 1) / *splits;
  *stages = *kbs_max < kQkvMaxStages ? *kbs_max : kQkvMaxStages;
}

// Shared memory of the tensor-core projection: weight ring, x tiles, the fp32
// partial tile, barriers (and 1024 bytes of alignment slack).
constexpr int kQkvABytes = kQkvTileM * kQkvTileK * 2;   // 16 KB weight tile
constexpr int kQkvBBytes = kQkvN * kQkvTileK * 2;       // 2 KB x tile
constexpr int kQkvPartBytes = kQkvN * kQkvTileM * 4;    // 8 KB fp32 partial tile
__host__ __device__ constexpr int qkv_mma_part_offset(int stages, int kbs_max) {
  return stages * kQkvABytes + kbs_max * kQkvBBytes;
}
__host__ __device__ constexpr int qkv_mma_bar_offset(int stages, int kbs_max) {
  return qkv_mma_part_offset(stages, kbs_max) + kQkvPartBytes;
}
__host__ __device__ constexpr int qkv_mma_smem_bytes(int stages, int kbs_max) {
  return qkv_mma_bar_offset(stages, kbs_max) + 256 + 1024;
}

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

// A CTA's coordinates: split s, key head h, batch b, first query head j0.
// The sub-groups of one split are adjacent in blockIdx.x, so they run in the
// same wave and the repeated key tiles come from L2.
struct CtaCoord {
  int s, h, b, j0;
};
__device__ inline CtaCoord cta_coord(const SplitParams& p) {
  CtaCoord c;
  c.s = blockIdx.x / p.hsplit;
  const int part = blockIdx.x - c.s * p.hsplit;
  c.h = blockIdx.y;
  c.b = blockIdx.z;
  c.j0 = (c.h * p.hsplit + part) * p.G;
  return c;
}

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
