// saga_kernels.cu - the SAGA + Atop-N decode-attention kernels for sm_100a.
//
// One decode step of one layer ("More Value per Key: Asymmetric Sparse
// Attention for Faster LLM Decoding"):
//   split kernel   : per (batch, key head, context split) CTA.  A TMA producer
//                    streams 128-token key tiles into a 128-byte-swizzled
//                    shared-memory ring; scores A = q K^T / sqrt(d) (eq. 2)
//                    for all query heads of the key head come from one
//                    tcgen05.mma per 16 dims (keys = M 128, queries = N,
//                    padded to 16) into TMEM; four epilogue warps compare
//                    against the Atop-N threshold (Atop-N step 1), compact
//                    the kept tokens with ballots, and accumulate the sparse
//                    softmax and value sum of eq. 7 online over the h_v
//                    value heads, writing one (max, sum, o) partial per split.
//   dump variant   : refresh steps (Atop-N step 2) - the same scores are
//                    written out (for groups of up to 4 heads, with counts
//                    of their top byte near the stale threshold).
//   select kernels : exact N-th largest score per row by radix selection
//                    (one CTA per row, or one thread-block cluster per row
//                    for a few long rows).
//   from-scores    : refresh steps - compare/gather from the dumped scores.
//   dense kernel   : every token kept, one value head per group - value
//                    tiles by TMA, online softmax per tile, no lists.
//   combine kernel : merges the split partials (log-sum-exp) into O.
//   append kernel  : writes the new token's key/value rows into the cache
//                    (when not fused into the attention kernels).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <utility>

#include "saga_device.cuh"
#include "saga_internal.h"

namespace saga {

// ============================================================================ helpers
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// N = 2 or 4 consecutive bf16 values (8- or 4-byte aligned) as floats.
template <int N>
__device__ __forceinline__ void load_bf16(const uint16_t* src, float (&v)[N]) {
  if constexpr (N == 4) {
    const uint2 raw = *reinterpret_cast<const uint2*>(src);
    v[0] = bf16_lo(raw.x);
    v[1] = bf16_hi(raw.x);
    v[2] = bf16_lo(raw.y);
    v[3] = bf16_hi(raw.y);
  } else {
    const uint32_t raw = *reinterpret_cast<const uint32_t*>(src);
    v[0] = bf16_lo(raw);
    v[1] = bf16_hi(raw);
  }
}

template <int N>
__device__ __forceinline__ void load_bf16_global(const uint16_t* src, float (&v)[N]) {
  if constexpr (N == 4) {
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(src));
    v[0] = bf16_lo(raw.x);
    v[1] = bf16_hi(raw.x);
    v[2] = bf16_lo(raw.y);
    v[3] = bf16_hi(raw.y);
  } else {
    const uint32_t raw = __ldg(reinterpret_cast<const uint32_t*>(src));
    v[0] = bf16_lo(raw);
    v[1] = bf16_hi(raw);
  }
}

// DPL bf16 values as one packed word (generic address: shared or global).
template <int N>
struct Bf16Pack;
template <>
struct Bf16Pack<4> {
  using T = uint2;
  static __device__ __forceinline__ T zero() { return make_uint2(0u, 0u); }
  static __device__ __forceinline__ void unpack(T r, float (&v)[4]) {
    v[0] = bf16_lo(r.x);
    v[1] = bf16_hi(r.x);
    v[2] = bf16_lo(r.y);
    v[3] = bf16_hi(r.y);
  }
};
template <>
struct Bf16Pack<2> {
  using T = uint32_t;
  static __device__ __forceinline__ T zero() { return 0u; }
  static __device__ __forceinline__ void unpack(T r, float (&v)[2]) {
    v[0] = bf16_lo(r);
    v[1] = bf16_hi(r);
  }
};

__device__ __forceinline__ bool named_bar_and(int id, int count, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return out != 0;
}



template <int NP>
__host__ __device__ constexpr uint32_t tmem_cols() { return (2 * NP <= 32) ? 32u : (2 * NP <= 64) ? 64u : 128u; }

// N of the scoring MMA: the group's query heads padded to the instruction's
// minimum of 16 (padding rows of q are zero; their columns are not read).
template <int NP>
__host__ __device__ constexpr int mma_n() { return NP < 16 ? 16 : NP; }

// TMEM accumulator buffers: the MMA may run this many tiles ahead of the
// epilogue (4 while they fit in 128 columns).
template <int NP>
__host__ __device__ constexpr int acc_bufs() { return mma_n<NP>() <= 32 ? 4 : 2; }

// ============================================================================ epilogue
// Each of the four epilogue warps owns 32 token rows of every tile (its TMEM
// lane quarter) and keeps its own online softmax, so no barrier couples the
// warps inside the tile loop.  Per tile a warp only compares its scores with
// the Atop-N thresholds (step 1) and, when some of its rows are kept, appends
// them (token, scores, head mask) to a warp-private list and starts copying
// their value rows into shared memory.  The softmax and the value sum of
// eq. 7 run per batch: when a list buffer is full (double-buffered, one
// refill behind) and at the end.  The four warps' partials are merged last.
constexpr int kBatch = 32;  // rows per list buffer

template <int NP>
struct WarpList {
  float sc[kBatch][NP];   // scores of the row for every head; overwritten by the weights
  uint64_t keep[kBatch];  // heads that keep the row
  int tok[kBatch];
};

template <int NP>
struct EpiShared {
  WarpList<NP> list[4][2];
  alignas(16) float tau[NP];  // Atop-N thresholds (+inf for padding heads)
  int vu[NP];                 // local value head of each query head of the group
  int hcnt[4][NP];            // counting mode: per-warp kept counts of the current tile
  int cnt_run[NP];            // counting mode: kept so far in this split
  int tail_buf[4][2];         // tail: each warp's unreduced list buffers ...
  int tail_n[4][2];           // ... and their row counts
};

// Bytes of value rows each warp stages per list buffer (2 KB at d = 64 with
// 16 heads per group, which lets two CTAs share an SM).
template <int D, int NP>
__host__ __device__ constexpr int vstage_warp_bytes() {
  return (NP >= 64 || (D == 64 && NP == 16)) ? 2048 : (D == 128 && NP <= 16) ? 8192 : 4096;
}

struct EpiArgs {
  const uint16_t* vgroup;  // V of the group's first value head, batch b
  int l_cap, G, hpv, nvh;
  int rcapw;  // rows per list buffer whose value rows are staged in shared memory
  int cpr;    // 16-byte chunks of one row over the group's value heads
  int hmul;   // ceil(65536 / hpv): (j * hmul) >> 16 == j / hpv for j < 64
  float scale;  // applied to a kept row's scores when it is listed (1 when they are scaled already)
};

// Per-lane online-softmax state: lane owns dims [lane*DPL, lane*DPL+DPL) of every head.
template <int D, int NP>
struct WarpAcc {
  static constexpr int DPL = D / 32;
  float m[NP];
  float l[NP];
  float o[NP][DPL];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      m[j] = -INFINITY;
      l[j] = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) o[j][e] = 0.f;
    }
  }
};

// A warp's list state: current buffer, its rows, and the full buffer waiting
// to be reduced (-1 if none).
struct ListState {
  int cur, n, pend, npend;
};

template <int D, int NP, int VSB = vstage_warp_bytes<D, NP>()>
__device__ __forceinline__ EpiArgs epi_args(const SplitParams& p, int b, int j0) {
  EpiArgs ea;
  const int v_base = (int)(((long long)j0 * p.h_v) / p.h_q);
  ea.vgroup = p.v_cache + ((size_t)b * p.h_v + v_base) * (size_t)p.l_cap * D;
  ea.l_cap = p.l_cap;
  ea.G = p.G;
  ea.hpv = p.hpv;
  ea.nvh = p.nvh;
  ea.rcapw = min(kBatch, VSB / (p.nvh * D * 2));
  ea.cpr = p.nvh * D / 8;
  ea.hmul = (65536 + p.hpv - 1) / p.hpv;
  ea.scale = p.scale;
  return ea;
}

// Thresholds: read from p.tau; every token kept (-inf) when p.tau is null
// (N covers every length); nothing compared in dump mode.  Padding heads keep
// nothing (+inf).  The load is separate from the shared-memory setup so that
// a kernel can issue all of its setup loads back to back.
// The smallest float x0 with fl(x0 * s) >= tv (s > 0): since x -> fl(x * s)
// is monotone, `x >= x0` decides exactly what `fl(x * s) >= tv` decides for
// every finite x, so a tile's raw dot products are compared without scaling
// them.  -inf / +inf map to themselves.
__device__ __forceinline__ bool scaled_ge(uint32_t k, float s, float tv) { return key_float(k) * s >= tv; }

__device__ float raw_threshold(float tv, float s) {
  if (tv == -INFINITY || tv == INFINITY) return tv;
  const float y = tv / s;
  if (y == INFINITY) return INFINITY;
  if (y == -INFINITY) return -INFINITY;
  const uint32_t kmin = float_key(-INFINITY), kmax = float_key(INFINITY);
  uint32_t k = float_key(y);
  for (int i = 0; i < 8 && k > kmin && scaled_ge(k - 1, s, tv); ++i) --k;
  for (int i = 0; i < 8 && k < kmax && !scaled_ge(k, s, tv); ++i) ++k;
  if (!(scaled_ge(k, s, tv) && (k == kmin || !scaled_ge(k - 1, s, tv)))) {
    // not found near tv / s: binary search over every float (predicate monotone in the key)
    uint32_t lo = kmin, hi = kmax;  // scaled_ge(kmax) holds: +inf * s = +inf
    while (lo < hi) {
      const uint32_t mid = lo + (hi - lo) / 2;
      if (scaled_ge(mid, s, tv)) hi = mid; else lo = mid + 1;
    }
    k = lo;
  }
  return key_float(k);
}

template <int NP>
__device__ __forceinline__ float load_tau(int et, const SplitParams& p, int b, int j0, bool compare) {
  float tv = INFINITY;
  if (compare && et < p.G) tv = p.tau != nullptr ? __ldg(p.tau + (size_t)b * p.h_q + j0 + et) : -INFINITY;
  return tv;
}

template <int NP>
__device__ __forceinline__ void epi_setup(EpiShared<NP>& es, int et, const SplitParams& p, float tv) {
  if (et < NP) {
    es.tau[et] = tv;
    es.vu[et] = et < p.G ? et / p.hpv : 0;
    es.cnt_run[et] = 0;
  }
}

// Atop-N step 1 for the lane's token: bit j set when query head j keeps it.
template <int NP>
__device__ __forceinline__ uint64_t keep_mask(const EpiShared<NP>& es, const float (&sc)[NP], bool valid) {
  if constexpr (NP <= 32) {
    uint32_t k32 = 0;
#pragma unroll
    for (int j4 = 0; j4 < NP / 4; ++j4) {
      const float4 tv = *reinterpret_cast<const float4*>(&es.tau[4 * j4]);
      k32 |= (uint32_t)(sc[4 * j4 + 0] >= tv.x) << (4 * j4 + 0);
      k32 |= (uint32_t)(sc[4 * j4 + 1] >= tv.y) << (4 * j4 + 1);
      k32 |= (uint32_t)(sc[4 * j4 + 2] >= tv.z) << (4 * j4 + 2);
      k32 |= (uint32_t)(sc[4 * j4 + 3] >= tv.w) << (4 * j4 + 3);
    }
    return valid ? (uint64_t)k32 : 0ull;
  }
  uint64_t keep = 0;
#pragma unroll
  for (int j4 = 0; j4 < NP / 4; ++j4) {
    const float4 tv = *reinterpret_cast<const float4*>(&es.tau[4 * j4]);
    if (sc[4 * j4 + 0] >= tv.x) keep |= 1ull << (4 * j4 + 0);
    if (sc[4 * j4 + 1] >= tv.y) keep |= 1ull << (4 * j4 + 1);
    if (sc[4 * j4 + 2] >= tv.z) keep |= 1ull << (4 * j4 + 2);
    if (sc[4 * j4 + 3] >= tv.w) keep |= 1ull << (4 * j4 + 3);
  }
  return valid ? keep : 0ull;
}

// One staged row of a list buffer into the warp's accumulators: every value
// head of the group is in shared memory, so the loads need no branch (heads
// that do not keep the row have weight 0).
template <int D, int NP>
__device__ __forceinline__ void staged_row(WarpAcc<D, NP>& acc, const EpiArgs& ea, const WarpList<NP>& li, int r,
                                           const uint16_t* vbuf) {
  constexpr int DPL = WarpAcc<D, NP>::DPL;
  float w[NP];
#pragma unroll
  for (int j4 = 0; j4 < NP / 4; ++j4) {
    const float4 v4 = *reinterpret_cast<const float4*>(&li.sc[r][4 * j4]);
    w[4 * j4 + 0] = v4.x;
    w[4 * j4 + 1] = v4.y;
    w[4 * j4 + 2] = v4.z;
    w[4 * j4 + 3] = v4.w;
  }
  const uint16_t* vrow = vbuf + (size_t)r * ea.nvh * D;
#pragma unroll
  for (int jl = 0; jl < NP; ++jl) {
    if (jl < ea.G) {
      float v[DPL];
      load_bf16<DPL>(vrow + ((jl * ea.hmul) >> 16) * D, v);
      acc.l[jl] += w[jl];
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc.o[jl][e] = fmaf(w[jl], v[e], acc.o[jl][e]);
    }
  }
}

// Softmax and value sum over list buffer bi (n rows) of this warp.
template <int D, int NP>
__device__ __forceinline__ void reduce_batch(EpiShared<NP>& es, WarpAcc<D, NP>& acc, const EpiArgs& ea, int q,
                                             int lane, int bi, int n, const uint16_t* vstage_w, bool newest_pending) {
  constexpr int DPL = WarpAcc<D, NP>::DPL;
  if (newest_pending) {
    asm volatile("cp.async.wait_group 1;" ::: "memory");  // the newest group belongs to the other buffer
  } else {
    cp_async_wait_all();
  }
  __syncwarp();
  WarpList<NP>& li = es.list[q][bi];
  const bool mine = lane < n;
  const uint64_t keep = mine ? li.keep[lane] : 0ull;
  float s[NP];
#pragma unroll
  for (int j4 = 0; j4 < NP / 4; ++j4) {
    float4 v = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    if (mine) v = *reinterpret_cast<const float4*>(&li.sc[lane][4 * j4]);
    s[4 * j4 + 0] = v.x;
    s[4 * j4 + 1] = v.y;
    s[4 * j4 + 2] = v.z;
    s[4 * j4 + 3] = v.w;
  }
  // batch maximum per head (one reduction over order-preserving keys); raise
  // the running maxima and rescale the running sums (warp-uniform branches)
#pragma unroll
  for (int jl = 0; jl < NP; ++jl) {
    const uint32_t k = ((keep >> jl) & 1ull) ? float_key(s[jl]) : 0u;
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, k);
    if (kmax != 0u) {
      const float tm = key_float(kmax);
      if (tm > acc.m[jl]) {
        const float f = (acc.m[jl] == -INFINITY) ? 0.f : __expf(acc.m[jl] - tm);
        acc.l[jl] *= f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc.o[jl][e] *= f;
        acc.m[jl] = tm;
      }
    }
  }
  // weights of the lane's row, written over its scores
  if (mine) {
#pragma unroll
    for (int j4 = 0; j4 < NP / 4; ++j4) {
      float4 w;
      w.x = ((keep >> (4 * j4 + 0)) & 1ull) ? __expf(s[4 * j4 + 0] - acc.m[4 * j4 + 0]) : 0.f;
      w.y = ((keep >> (4 * j4 + 1)) & 1ull) ? __expf(s[4 * j4 + 1] - acc.m[4 * j4 + 1]) : 0.f;
      w.z = ((keep >> (4 * j4 + 2)) & 1ull) ? __expf(s[4 * j4 + 2] - acc.m[4 * j4 + 2]) : 0.f;
      w.w = ((keep >> (4 * j4 + 3)) & 1ull) ? __expf(s[4 * j4 + 3] - acc.m[4 * j4 + 3]) : 0.f;
      *reinterpret_cast<float4*>(&li.sc[lane][4 * j4]) = w;
    }
  }
  __syncwarp();
  // staged rows in groups (their loads are independent, so a group's are in
  // flight together), then any rows that did not fit the staging buffer
  const uint16_t* vbuf = vstage_w + (size_t)bi * ea.rcapw * ea.nvh * D + lane * DPL;
  const int ns = min(n, ea.rcapw);
  constexpr int RU = NP <= 8 ? 4 : (NP == 16 ? 2 : 1);
  int r = 0;
  for (; r + RU <= ns; r += RU) {
#pragma unroll
    for (int k = 0; k < RU; ++k) staged_row<D, NP>(acc, ea, li, r + k, vbuf);
  }
  for (; r < ns; ++r) staged_row<D, NP>(acc, ea, li, r, vbuf);
  for (; r < n; ++r) {
    float w[NP];
#pragma unroll
    for (int j4 = 0; j4 < NP / 4; ++j4) {
      const float4 v4 = *reinterpret_cast<const float4*>(&li.sc[r][4 * j4]);
      w[4 * j4 + 0] = v4.x;
      w[4 * j4 + 1] = v4.y;
      w[4 * j4 + 2] = v4.z;
      w[4 * j4 + 3] = v4.w;
    }
    const uint16_t* vrow = ea.vgroup + (size_t)li.tok[r] * D + lane * DPL;
#pragma unroll
    for (int jl = 0; jl < NP; ++jl) {
      if (w[jl] != 0.f) {  // same value in every lane
        float v[DPL];
        load_bf16_global<DPL>(vrow + (size_t)((jl * ea.hmul) >> 16) * ea.l_cap * D, v);
        acc.l[jl] += w[jl];
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc.o[jl][e] = fmaf(w[jl], v[e], acc.o[jl][e]);
      }
    }
  }
  __syncwarp();
}

// Appends the warp's kept rows of one tile to its list (reducing a full
// buffer one refill later) and starts staging their value rows.
template <int D, int NP>
__device__ __forceinline__ void append_rows(EpiShared<NP>& es, WarpAcc<D, NP>& acc, const EpiArgs& ea, ListState& ls,
                                            int q, int lane, uint32_t bal, uint64_t keep, const float (&sc)[NP],
                                            int tok, uint16_t* vstage_w) {
  const int nnew = __popc(bal);
  if (ls.n + nnew > kBatch) {
    if (ls.pend >= 0) reduce_batch<D, NP>(es, acc, ea, q, lane, ls.pend, ls.npend, vstage_w, true);
    ls.pend = ls.cur;
    ls.npend = ls.n;
    ls.cur ^= 1;
    ls.n = 0;
  }
  WarpList<NP>& li = es.list[q][ls.cur];
  if (keep != 0ull) {
    const int pos = ls.n + __popc(bal & ((1u << lane) - 1u));
    li.tok[pos] = tok;
    li.keep[pos] = keep;
#pragma unroll
    for (int j4 = 0; j4 < NP / 4; ++j4)
      *reinterpret_cast<float4*>(&li.sc[pos][4 * j4]) =
          make_float4(sc[4 * j4 + 0] * ea.scale, sc[4 * j4 + 1] * ea.scale, sc[4 * j4 + 2] * ea.scale,
                      sc[4 * j4 + 3] * ea.scale);
  }
  __syncwarp();
  // value rows (every value head of the group) of the new list entries:
  // staged in shared memory while the buffer has room, otherwise warmed in L2
  const int r0 = ls.n, r1 = ls.n + nnew;
  const int rs = min(r1, ea.rcapw);
  for (int it = lane; it < max(0, rs - r0) * ea.cpr; it += 32) {
    const int ri = r0 + it / ea.cpr, ch = it % ea.cpr;
    const int u = ch / (D / 8), cc = ch - u * (D / 8);
    cp_async16(vstage_w + (((size_t)ls.cur * ea.rcapw + ri) * ea.nvh + u) * D + cc * 8,
                 ea.vgroup + ((size_t)u * ea.l_cap + li.tok[ri]) * D + cc * 8);
  }
  for (int it = lane; it < max(0, r1 - max(r0, rs)) * ea.nvh * (D / 64); it += 32) {
    const int per = ea.nvh * (D / 64);
    const int ri = max(r0, rs) + it / per, rem = it % per;
    const int u = rem / (D / 64), line = rem % (D / 64);
    const char* src = reinterpret_cast<const char*>(ea.vgroup + ((size_t)u * ea.l_cap + li.tok[ri]) * D) + line * 128;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(src));
  }
  cp_async_commit();
  ls.n = r1;
}

// Counting mode (kept counts and ascending index lists requested): the four
// warps go through each tile together; per-head ballots give each kept
// token its position in the split's list.
template <int NP>
__device__ __forceinline__ void count_tile(EpiShared<NP>& es, uint64_t keep, int q, int lane, int et, int tok,
                                           const SplitParams& p, int b, int j0, int chunk_start) {
#pragma unroll
  for (int jl = 0; jl < NP; ++jl) {
    if (jl < p.G) {
      const uint32_t bl = __ballot_sync(0xffffffffu, (keep >> jl) & 1ull);
      if (lane == 0) es.hcnt[q][jl] = __popc(bl);
    }
  }
  named_bar_sync(1, kEpiThreads);
  if (p.idxbuf != nullptr) {
#pragma unroll
    for (int jl = 0; jl < NP; ++jl) {
      if (jl < p.G) {
        const bool kb = (keep >> jl) & 1ull;
        const uint32_t bl = __ballot_sync(0xffffffffu, kb);
        if (kb) {
          int off = es.cnt_run[jl];
          for (int qq = 0; qq < q; ++qq) off += es.hcnt[qq][jl];
          off += __popc(bl & ((1u << lane) - 1u));
          p.idxbuf[((size_t)b * p.h_q + j0 + jl) * p.l_cap + chunk_start + off] = tok;
        }
      }
    }
  }
  named_bar_sync(1, kEpiThreads);
  if (et < p.G) es.cnt_run[et] += es.hcnt[0][et] + es.hcnt[1][et] + es.hcnt[2][et] + es.hcnt[3][et];
}

// Per tile of one warp: threshold compare, optional counting, list append.
template <int D, int NP>
__device__ __forceinline__ void tile_epilogue(EpiShared<NP>& es, WarpAcc<D, NP>& acc, const EpiArgs& ea,
                                              ListState& ls, int q, int lane, int et, const float (&sc)[NP], int tok,
                                              bool valid, bool counting, const SplitParams& p, int b, int j0,
                                              int chunk_start, uint16_t* vstage_w) {
  const uint64_t keep = keep_mask<NP>(es, sc, valid);
  const uint32_t bal = __ballot_sync(0xffffffffu, keep != 0ull);
  if (counting) count_tile<NP>(es, keep, q, lane, et, tok, p, b, j0, chunk_start);
  if (bal != 0u) append_rows<D, NP>(es, acc, ea, ls, q, lane, bal, keep, sc, tok, vstage_w);
}

// Tail of a split: merges the four warps' running (m, l, o) with the rows
// still waiting, unreduced, in their lists, and writes the split's partial.
// Each warp publishes its state (in mrg: 4 * NP * (D + 2) floats, 16-byte
// aligned) and its list descriptors.  After one barrier the unreduced rows
// of all warps form one pool; each warp takes a block of contiguous heads
// and works on them together: its lanes first hold one pool row each
// (weights, one max reduction per head), then the columns while the rows
// are accumulated from shuffled weights.
// Deterministic (fixed order in every sum).
template <int D, int NP>
__host__ __device__ constexpr int merge_floats() { return 4 * NP * (D + 2); }

template <int D, int NP, int VSB = vstage_warp_bytes<D, NP>()>
__device__ __forceinline__ void tail_merge(EpiShared<NP>& es, float* mrg, const WarpAcc<D, NP>& acc,
                                           const ListState& ls, const EpiArgs& ea, const uint16_t* vstage, int q,
                                           int lane, int et, const SplitParams& p, int b, int j0, int s,
                                           bool drop_lists) {
  constexpr int DPL = WarpAcc<D, NP>::DPL;
  constexpr int REG = NP * (D + 2);
  constexpr int VWE = VSB;  // elements of one warp's staging area (two buffers)
  float* mine = mrg + q * REG;                  // m[NP], l[NP], o[NP][D]
  if (lane == 0) {
#pragma unroll
    for (int j4 = 0; j4 < NP / 4; ++j4) {
      *reinterpret_cast<float4*>(&mine[4 * j4]) =
          make_float4(acc.m[4 * j4], acc.m[4 * j4 + 1], acc.m[4 * j4 + 2], acc.m[4 * j4 + 3]);
      *reinterpret_cast<float4*>(&mine[NP + 4 * j4]) =
          make_float4(acc.l[4 * j4], acc.l[4 * j4 + 1], acc.l[4 * j4 + 2], acc.l[4 * j4 + 3]);
    }
    es.tail_buf[q][0] = ls.pend & 1;
    es.tail_n[q][0] = (ls.pend >= 0 && !drop_lists) ? ls.npend : 0;
    es.tail_buf[q][1] = ls.cur & 1;
    es.tail_n[q][1] = drop_lists ? 0 : ls.n;
  }
#pragma unroll
  for (int jl = 0; jl < NP; ++jl) {
    float* dst = &mine[2 * NP + jl * D + lane * DPL];
    if constexpr (DPL == 4) {
      *reinterpret_cast<float4*>(dst) = make_float4(acc.o[jl][0], acc.o[jl][1], acc.o[jl][2], acc.o[jl][3]);
    } else {
      *reinterpret_cast<float2*>(dst) = make_float2(acc.o[jl][0], acc.o[jl][1]);
    }
  }
  cp_async_wait_all();  // this thread's staged value rows; the barrier publishes everyone's
  named_bar_sync(1, kEpiThreads);

  // the unreduced rows of all warps form one pool: (warp, buffer) lists in order
  int off[9];
  off[0] = 0;
#pragma unroll
  for (int wk = 0; wk < 8; ++wk) off[wk + 1] = off[wk] + es.tail_n[wk >> 1][wk & 1];
  const int npool = off[8];
  const size_t row0 = (size_t)b * p.h_q + j0;
  // warp q takes the contiguous heads [q*HB, q*HB + HB) (with h_q/h_v query
  // heads per value head these usually share one value head) and works on
  // them together: one pass over the pool serves all of them
  constexpr int NH = (NP + 3) / 4;
  const int HB = (p.G + 3) / 4;
  const int h0 = q * HB;
  float M[NH], mwv[NH][4];
  int u[NH];
  bool hv[NH];
#pragma unroll
  for (int hh = 0; hh < NH; ++hh) {
    const int jl = h0 + hh;
    hv[hh] = hh < HB && jl < p.G;
    u[hh] = hv[hh] ? (jl * ea.hmul) >> 16 : 0;
    M[hh] = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      mwv[hh][w] = hv[hh] ? mrg[w * REG + jl] : -INFINITY;
      M[hh] = fmaxf(M[hh], mwv[hh][w]);
    }
  }
  // lane k of a chunk holds pool row base + k: its list, row, keep mask, scores
  for (int base = 0; base < npool; base += 32) {
    const int k = base + lane;
    uint64_t keep = 0ull;
    int wk = 0, r = k;
    if (k < npool) {
#pragma unroll
      for (int i = 1; i < 8; ++i)
        if (k >= off[i]) {
          wk = i;
          r = k - off[i];
        }
      keep = es.list[wk >> 1][es.tail_buf[wk >> 1][wk & 1]].keep[r];
    }
    const WarpList<NP>& li = es.list[wk >> 1][es.tail_buf[wk >> 1][wk & 1]];
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
      const int jl = h0 + hh;
      const uint32_t kk = (hv[hh] && ((keep >> jl) & 1ull)) ? float_key(li.sc[r][jl]) : 0u;
      const uint32_t kmax = __reduce_max_sync(0xffffffffu, kk);
      if (kmax != 0u) M[hh] = fmaxf(M[hh], key_float(kmax));
    }
  }
  float o[NH][DPL], lsum[NH];
#pragma unroll
  for (int hh = 0; hh < NH; ++hh) {
    const int jl = h0 + hh;
    lsum[hh] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) o[hh][e] = 0.f;
    if (hv[hh] && M[hh] != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float f = (mwv[hh][w] == -INFINITY) ? 0.f : __expf(mwv[hh][w] - M[hh]);
        lsum[hh] = fmaf(f, mrg[w * REG + NP + jl], lsum[hh]);
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[hh][e] = fmaf(f, mrg[w * REG + 2 * NP + jl * D + lane * DPL + e], o[hh][e]);
      }
    }
  }
  for (int base = 0; base < npool; base += 32) {
    // lane k: its pool row's weights and where its value rows are (shared
    // memory offset of value head 0 of the group, or -(token + 1) for a row
    // that was not staged)
    const int k = base + lane;
    float wgt[NH];
    int loc = 0;
    {
      uint64_t keep = 0ull;
      int wk = 0, r = k, bi = 0;
      if (k < npool) {
#pragma unroll
        for (int i = 1; i < 8; ++i)
          if (k >= off[i]) {
            wk = i;
            r = k - off[i];
          }
        bi = es.tail_buf[wk >> 1][wk & 1];
        keep = es.list[wk >> 1][bi].keep[r];
      }
      const WarpList<NP>& li = es.list[wk >> 1][bi];
#pragma unroll
      for (int hh = 0; hh < NH; ++hh) {
        const int jl = h0 + hh;
        const bool kept = hv[hh] && ((keep >> jl) & 1ull);
        wgt[hh] = kept ? __expf(li.sc[r][jl] - M[hh]) : 0.f;
        lsum[hh] += warp_sum(wgt[hh]);
      }
      if (k < npool) loc = r < ea.rcapw ? (wk >> 1) * VWE + (bi * ea.rcapw + r) * ea.nvh * D : -(li.tok[r] + 1);
    }
    // rows in groups of RG: every value load of a group (shared memory for
    // staged rows, L2 for the others) is issued before the group's sums, so
    // their latencies overlap; the sums keep the row order
    using PK = Bf16Pack<DPL>;
    constexpr int RG = NH <= 4 ? 4 : 2;
    const int nrow = min(32, npool - base);
    for (int i0 = 0; i0 < nrow; i0 += RG) {
      typename PK::T raw[RG][NH];
      float wv[RG][NH];
#pragma unroll
      for (int k = 0; k < RG; ++k) {
        const int i = i0 + k;
        const int li_loc = __shfl_sync(0xffffffffu, loc, i & 31);
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          const float w = __shfl_sync(0xffffffffu, wgt[hh], i & 31);
          wv[k][hh] = i < nrow ? w : 0.f;
          const uint16_t* src = li_loc >= 0
                                    ? vstage + li_loc + u[hh] * D + lane * DPL
                                    : ea.vgroup + ((size_t)u[hh] * ea.l_cap + (size_t)(-li_loc - 1)) * D + lane * DPL;
          raw[k][hh] = PK::zero();
          if (wv[k][hh] != 0.f) raw[k][hh] = *reinterpret_cast<const typename PK::T*>(src);
        }
      }
#pragma unroll
      for (int k = 0; k < RG; ++k) {
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          if (wv[k][hh] != 0.f) {  // warp-uniform
            float v[DPL];
            PK::unpack(raw[k][hh], v);
#pragma unroll
            for (int e = 0; e < DPL; ++e) o[hh][e] = fmaf(wv[k][hh], v[e], o[hh][e]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int hh = 0; hh < NH; ++hh) {
    if (!hv[hh]) continue;
    const int jl = h0 + hh;
    float* dst = &p.part_o[((row0 + jl) * p.s_cap + s) * D + lane * DPL];
    if constexpr (DPL == 4) {
      *reinterpret_cast<float4*>(dst) = make_float4(o[hh][0], o[hh][1], o[hh][2], o[hh][3]);
    } else {
      *reinterpret_cast<float2*>(dst) = make_float2(o[hh][0], o[hh][1]);
    }
    if (lane == 0) {
      p.part_m[(row0 + jl) * p.s_cap + s] = M[hh];
      p.part_l[(row0 + jl) * p.s_cap + s] = lsum[hh];
      p.part_cnt[(row0 + jl) * p.s_cap + s] = es.cnt_run[jl];
    }
  }
}

// ============================================================================ split kernel
constexpr int kSmemLimit = 232448;  // dynamic shared memory one CTA may use on sm_100
constexpr int kSmemHalf = 115712;   // per CTA when two CTAs share an SM (233472 / 2 minus the 1 KB reserve)

template <int D, int NP, bool UMMA>
struct SplitSmem {
  static constexpr int NATOM = D / 64;
  static constexpr int STAGE_BYTES = kTile * D * 2;
  static constexpr int QBYTES = UMMA ? NATOM * mma_n<NP>() * 128 : NP * D * 4;
  static constexpr int QPAD = ((QBYTES + 1023) / 1024) * 1024;
  static constexpr int EPI_BYTES = ((int)sizeof(EpiShared<NP>) + 127) / 128 * 128;
  static constexpr int VST_BYTES = 4 * 2 * vstage_warp_bytes<D, NP>();
  // key-tile ring: 4 tiles of 32 KB at d = 128 or 6 of 16 KB at d = 64 cover
  // the load latency; fewer where the epilogue's buffers leave less room.
  // At d = 64, when 4 tiles of 16 KB fit in half of the SM's shared memory,
  // the ring takes 4 so that two CTAs share an SM (twice the epilogue warps
  // to hide latency, as many bytes in flight).
  static constexpr int NSTAGE_MAX = D == 128 ? 4 : 6;
  static constexpr int FIXED = QPAD + EPI_BYTES + VST_BYTES + (2 * NSTAGE_MAX + 2 * acc_bufs<NP>() + 2) * 8 + 16 + 1024;
  static constexpr int NSTAGE_FIT = (kSmemLimit - FIXED) / STAGE_BYTES;
  static constexpr int NSTAGE_HALF = (kSmemHalf - FIXED) / STAGE_BYTES;
  static constexpr bool TWO = D == 64 && NSTAGE_HALF >= 4;  // 2 x 32 KB at d = 128 measured slower
  static constexpr int NSTAGE_TWO = NSTAGE_HALF < 4 ? NSTAGE_HALF : 4;
  static constexpr int NSTAGE = TWO ? NSTAGE_TWO : (NSTAGE_FIT < NSTAGE_MAX ? NSTAGE_FIT : NSTAGE_MAX);
  static constexpr int CTAS_PER_SM = TWO ? 2 : 1;  // also bounds the registers (<= 170 for two)
  static_assert(NSTAGE >= 3 || (TWO && NSTAGE >= 2), "key-tile ring too shallow");
  static constexpr int Q_OFF = NSTAGE * STAGE_BYTES;
  static constexpr int EPI_OFF = Q_OFF + QPAD;
  static constexpr int VST_OFF = EPI_OFF + EPI_BYTES;
  static constexpr int BAR_OFF = VST_OFF + VST_BYTES;
  static constexpr int NBARS = 2 * NSTAGE + 2 * acc_bufs<NP>() + 2;  // + fin, + the test hook's barrier
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
  static_assert(ALLOC <= kSmemLimit, "shared memory over the per-CTA limit");
  static_assert(!TWO || ALLOC <= kSmemHalf, "two CTAs per SM must fit in half the shared memory");
  static_assert(merge_floats<D, NP>() * 4 <= NSTAGE * STAGE_BYTES, "merge buffer must fit in the key stages");
  static_assert(NP > kDumpHistMaxNp || NP * 256 * 4 <= (int)sizeof(WarpList<NP>) * 8,
                "dump counts must fit in the warp lists");
};

// Fused append: row pos of key head h and of the group's value heads, from
// k_new / v_new.  With h_v < h_k several key heads share a value head and
// each of their splits writes the same bytes.
template <int D>
__device__ __forceinline__ void append_new_rows(const SplitParams& p, int b, int h, int j0, int pos) {
  constexpr int C = D / 8;  // 16-byte chunks per row
  const int v_base = (int)(((long long)j0 * p.h_v) / p.h_q);
  const int n = (1 + p.nvh) * C;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int r = i / C, c = i % C;
    if (r == 0) {
      const size_t kh = (size_t)b * p.h_k + h;
      const uint4 v = reinterpret_cast<const uint4*>(p.k_new + kh * D)[c];
      reinterpret_cast<uint4*>(p.k_cache_w + (kh * p.l_cap + pos) * D)[c] = v;
    } else {
      const size_t vh = (size_t)b * p.h_v + v_base + r - 1;
      const uint4 v = reinterpret_cast<const uint4*>(p.v_new + vh * D)[c];
      reinterpret_cast<uint4*>(p.v_cache_w + (vh * p.l_cap + pos) * D)[c] = v;
    }
  }
  fence_proxy_async_global();
}

// One key tile: 128 rows (or the rows left in the split, as 32-row boxes)
// of every 64-column swizzle atom, into stage t % NSTAGE.
template <int NATOM, int NSTAGE, int STAGE_BYTES>
__device__ __forceinline__ void issue_key_tile(int t, int start, int end, int row_base, uint8_t* kst, uint64_t* full,
                                               const CUtensorMap* tmap_full, const CUtensorMap* tmap_part) {
  const int stage = t % NSTAGE;
  const int r0 = start + t * kTile;
  const int rows = min(kTile, end - r0);
  uint8_t* dst = kst + stage * STAGE_BYTES;
  if (rows == kTile) {
    mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
#pragma unroll
    for (int a = 0; a < NATOM; ++a) tma_load_2d(dst + a * 16384, tmap_full, &full[stage], a * 64, row_base + r0);
  } else {
    const int nsub = (rows + kUnit - 1) / kUnit;
    mbar_arrive_expect_tx(&full[stage], nsub * kUnit * 128 * NATOM);
    for (int i = 0; i < nsub; ++i)
#pragma unroll
      for (int a = 0; a < NATOM; ++a)
        tma_load_2d(dst + a * 16384 + i * kUnit * 128, tmap_part, &full[stage], a * 64, row_base + r0 + i * kUnit);
  }
}

// Warp roles: 0 = TMA producer, 1 = tcgen05 MMA issuer, 2..5 = epilogue
// (one thread per token row of a tile).
template <int D, int NP, bool UMMA, bool DUMP>
__global__ void __launch_bounds__(192, SplitSmem<D, NP, UMMA>::CTAS_PER_SM)
    saga_split_kernel(const __grid_constant__ CUtensorMap tmap_full, const __grid_constant__ CUtensorMap tmap_part,
                      const SplitParams p) {
  static_assert(UMMA, "scores come from tcgen05 for every group size");
  // dump of a small group: also count the top byte of the scores near the stale threshold
  constexpr bool DHIST = DUMP && NP <= kDumpHistMaxNp;
  using SM = SplitSmem<D, NP, UMMA>;
  constexpr int NATOM = SM::NATOM;
  constexpr int NSTAGE = SM::NSTAGE;
  constexpr int STAGE_BYTES = SM::STAGE_BYTES;
  constexpr int NPM = mma_n<NP>();
  constexpr int NACC = acc_bufs<NP>();
  constexpr uint32_t TMEM_COLS = NACC * NPM <= 32 ? 32u : NACC * NPM <= 64 ? 64u : NACC * NPM <= 128 ? 128u : 256u;
  constexpr uint32_t IDESC = umma_idesc_bf16(128, NPM);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kst = smem;
  uint8_t* qsm = smem + SM::Q_OFF;
  EpiShared<NP>& es = *reinterpret_cast<EpiShared<NP>*>(smem + SM::EPI_OFF);
  uint16_t* vstage = reinterpret_cast<uint16_t*>(smem + SM::VST_OFF);
  uint32_t* hist = reinterpret_cast<uint32_t*>(&es.list[0][0]);  // DHIST: [NP][256]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::BAR_OFF);
  uint64_t* empty = full + NSTAGE;
  uint64_t* accf = empty + NSTAGE;
  uint64_t* acce = accf + NACC;
  uint64_t* fin = acce + NACC;
  uint64_t* never = fin + 1;  // test hook: a barrier nothing arrives at
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::MISC_OFF + 4);

  const CtaCoord cc = cta_coord(p);
  const int s = cc.s, h = cc.h, b = cc.b;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = cc.j0;
  const int row_base = (b * p.h_k + h) * p.l_cap;  // first cache row of this (batch, key head)

  // ---------------------------------------------------------------- setup before the dependency wait
  // Nothing used here is written by a preceding kernel: barriers, TMEM, the
  // tensor maps, and an L2 prefetch of the key rows this split can cover
  // whatever the length (a prefetch moves no values, so it races with
  // nothing).
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], UMMA ? 1 : 4);
    }
    for (int i = 0; i < NACC; ++i) {
      mbar_init(&accf[i], 1);
      mbar_init(&acce[i], 4);
    }
    mbar_init(fin, 1);
    mbar_init(never, 1);
    mbar_init_fence();
    tma_prefetch_desc(&tmap_full);
    tma_prefetch_desc(&tmap_part);
    int pst, pcap;
    split_cap_range(p.seq_len, p.nsplit, s, p.l_cap, &pst, &pcap);
    // as much of the split as fits the grid's share of 48 MB of L2 (the
    // previous kernel's tail leaves DRAM idle; more would evict itself)
    const long long ncta = (long long)gridDim.x * gridDim.y * gridDim.z;
    const int cap_rows = max(kTile, (int)(((48ll << 20) / ncta) / (D * 2)) / kTile * kTile);
    const int pend = min(pcap, pst + cap_rows);
    const uint16_t* kb = p.k_cache + (size_t)row_base * D;
    for (int r = pst; r < pend; r += kTile) prefetch_l2_bulk(kb + (size_t)r * D, (uint32_t)(min(kTile, pend - r) * D * 2));
  } else if (warp == 2) {
    // the group's query rows and thresholds, read right after the wait
    const char* qg = reinterpret_cast<const char*>(p.q + ((size_t)b * p.h_q + j0) * D);
    for (int i = lane; i < p.G * D * 2 / 128; i += 32) prefetch_l2_line(qg + 128 * i);
    if (lane == 0 && p.tau != nullptr && !DUMP) prefetch_l2_line(p.tau + (size_t)b * p.h_q + j0);
  }
  if (UMMA && warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();

  // ---------------------------------------------------------------- setup after it
  // The global reads of this setup (q, the thresholds, the length) are issued
  // back to back so that their latencies overlap.
  constexpr int QCH = UMMA ? NATOM * NPM * 8 : NP * D / 8;  // 16-byte chunks of the group's q (padded heads)
  constexpr int QV = (QCH + kEpiThreads - 1) / kEpiThreads;
  const int eth = threadIdx.x - 64;  // epilogue thread (warps 2..5)
  uint4 qv[QV];
  float tv = INFINITY;
  if (warp >= 2) {
#pragma unroll
    for (int k = 0; k < QV; ++k) {
      const int i = eth + k * kEpiThreads;
      int n, col;
      if (UMMA) {
        n = (i / 8) % NPM;
        col = (i / (NPM * 8)) * 64 + (i % 8) * 8;
      } else {
        n = i / (D / 8);
        col = (i % (D / 8)) * 8;
      }
      qv[k] = make_uint4(0, 0, 0, 0);
      if (i < QCH && n < p.G)
        qv[k] = __ldg(reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.h_q + j0 + n) * D + col));
    }
    tv = load_tau<NP>(eth, p, b, j0, !DUMP);
    if (DHIST && p.hist_out != nullptr && p.tau != nullptr && eth < p.G) tv = __ldg(p.tau + (size_t)b * p.h_q + j0 + eth);
  }
  // the epilogue compares raw dot products (scaled only once listed)
  if (!DUMP && warp >= 2 && eth < NP) tv = raw_threshold(tv, p.scale);
  const int L = device_seq_len(p.seq_len_dev, p.seq_len, p.l_cap, (s == 0 && h == 0 && b == 0) ? p.status : nullptr);
  int start, end;
  split_range(p.seq_len, p.nsplit, s, L, &start, &end);
  const int ntiles = (end - start + kTile - 1) / kTile;
  // fused append: the split holding row L - 1 writes the new key/value rows;
  // its tile holding that row is loaded only after the barrier below
  const bool owner = p.k_new != nullptr && start <= L - 1 && L - 1 < end;
  if (owner) append_new_rows<D>(p, b, h, j0, L - 1);
  int issued = 0;  // producer: tiles issued
  if (threadIdx.x == 0) {
    for (; issued < ntiles && issued < NSTAGE; ++issued) {
      if (owner && L - 1 < start + (issued + 1) * kTile) break;
      issue_key_tile<NATOM, NSTAGE, STAGE_BYTES>(issued, start, end, row_base, kst, full, &tmap_full, &tmap_part);
    }
  }
  if (warp >= 2) {
    epi_setup<NP>(es, eth, p, tv);
#pragma unroll
    for (int k = 0; k < QV; ++k) {
      const int i = eth + k * kEpiThreads;
      if (i < QCH) {
        if (UMMA) {
          // q as the K-major B operand in the 128-byte swizzle layout; rows >= G are zero
          const int a = i / (NPM * 8), n = (i / 8) % NPM, c = i % 8;
          *reinterpret_cast<uint4*>(qsm + a * NPM * 128 + n * 128 + ((c ^ (n & 7)) << 4)) = qv[k];
        } else {
          float* qf = reinterpret_cast<float*>(qsm) + (i / (D / 8)) * D + (i % (D / 8)) * 8;
          *reinterpret_cast<float4*>(qf) = make_float4(bf16_lo(qv[k].x), bf16_hi(qv[k].x), bf16_lo(qv[k].y),
                                                       bf16_hi(qv[k].y));
          *reinterpret_cast<float4*>(qf + 4) = make_float4(bf16_lo(qv[k].z), bf16_hi(qv[k].z), bf16_lo(qv[k].w),
                                                           bf16_hi(qv[k].w));
        }
      }
    }
    if (DHIST)
      for (int i = eth; i < NP * 256; i += kEpiThreads) hist[i] = 0u;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = UMMA ? *tmem_slot : 0u;

  // ---------------------------------------------------------------- roles
  if (warp == 0) {
    if (lane == 0) {
      if (owner) fence_proxy_async_global();  // the appended rows (written before the barrier) reach TMA
      for (int t = issued; t < ntiles; ++t) {
        const int stage = t % NSTAGE, round = t / NSTAGE;
        if (round > 0 && !mbar_wait(&empty[stage], (round - 1) & 1, abort_flag)) break;
        issue_key_tile<NATOM, NSTAGE, STAGE_BYTES>(t, start, end, row_base, kst, full, &tmap_full, &tmap_part);
        issued = t + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (UMMA && lane == 0) {
      for (int t = 0; t < ntiles; ++t) {
        const int stage = t % NSTAGE, round = t / NSTAGE;
        if (!mbar_wait(&full[stage], round & 1, abort_flag)) break;
        const int abuf = t % NACC;
        if (t >= NACC && !mbar_wait(&acce[abuf], ((t / NACC) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(kst + stage * STAGE_BYTES);
        const uint32_t b0 = smem_u32(qsm);
        const uint32_t d_tmem = tmem_base + abuf * NPM;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t aa = a0 + (k >> 2) * 16384 + (k & 3) * 32;
          const uint32_t bb = b0 + (k >> 2) * NPM * 128 + (k & 3) * 32;
          umma_bf16(d_tmem, umma_sdesc_sw128(aa), umma_sdesc_sw128(bb), IDESC, k > 0 ? 1u : 0u);
        }
        umma_commit(&empty[stage]);
        umma_commit(&accf[abuf]);
      }
      // drain: every MMA issued by this thread has completed once `fin` fires
      umma_commit(fin);
      if (!mbar_wait_drain(fin, 0)) *abort_flag = 1;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;
    const int q = warp & 3;           // TMEM lane quarter: rows 32q .. 32q+31 of every tile
    const int erow = 32 * q + lane;
    const bool counting = p.want_counts != 0;
    const EpiArgs ea = epi_args<D, NP>(p, b, j0);
    uint16_t* vstage_w = vstage + (size_t)q * 2 * (vstage_warp_bytes<D, NP>() / 2);
    WarpAcc<D, NP> acc;
    acc.init();
    ListState ls{0, 0, -1, 0};
    const size_t srow = ((size_t)b * p.h_q + j0) * (size_t)p.ld_scores;
    // DHIST: the select needs exact counts only from the bin of the N-th largest up, so the top-byte
    // bins from two below the stale threshold's bin up are counted (a bin spans two binades, so for a
    // positive threshold that reaches scores 16 to 64 times smaller); the select checks that the
    // counted bins hold N scores and otherwise counts the row itself
    uint32_t bfl[NP];
#pragma unroll
    for (int jl = 0; jl < NP; ++jl) {
      bfl[jl] = 0u;
      if (DHIST && p.hist_floor != 0 && jl < p.G) {
        const float ts = es.tau[jl];  // the stale threshold (scaled, as the dumped scores)
        if (ts != -INFINITY && ts == ts) {
          const uint32_t tb = float_key(ts) >> 24;
          bfl[jl] = tb > 2u ? tb - 2u : 0u;
        }
      }
    }
    int t = 0;
    if (!DUMP && p.test_wait_ns != 0u) {
      bool ok = __all_sync(0xffffffffu, mbar_wait(never, 0, abort_flag, p.test_wait_ns));
      if (counting) ok = named_bar_and(1, kEpiThreads, ok);
      if (!ok) t = -1;  // skips the tile loop; the tail drops the (empty) lists
    }
    for (; t >= 0 && t < ntiles; ++t) {
      float sc[NP];
      bool ok;
      {
        const int abuf = t % NACC;
        ok = __all_sync(0xffffffffu, mbar_wait(&accf[abuf], (t / NACC) & 1, abort_flag));
        if (counting) ok = named_bar_and(1, kEpiThreads, ok);  // warps leave together (barriers below)
        if (!ok) break;
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(abuf * NPM);
        if constexpr (NP >= 16) {
#pragma unroll
          for (int i = 0; i < NP / 16; ++i) tmem_ld16(taddr + 16 * i, sc + 16 * i);
        } else {
          float all[16];
          tmem_ld16(taddr, all);
#pragma unroll
          for (int i = 0; i < NP; ++i) sc[i] = all[i];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[abuf]);
      }
      if (DUMP) {
#pragma unroll
        for (int n = 0; n < NP; ++n) sc[n] *= p.scale;
      }
      const int tok = start + t * kTile + erow;
      const bool valid = tok < end;
      if (DUMP) {
#pragma unroll
        for (int jl = 0; jl < NP; ++jl) {
          if (jl < p.G) {
            if (valid) p.scores_out[srow + (size_t)jl * p.ld_scores + tok] = sc[jl];
            if (DHIST && p.hist_out != nullptr) {
              const uint32_t bin = float_key(sc[jl]) >> 24;
              const bool counted = valid && bin >= bfl[jl];
              if (__any_sync(0xffffffffu, counted)) {
                const uint32_t peers = __match_any_sync(0xffffffffu, counted ? bin : 256u);
                if (counted && lane == __ffs(peers) - 1) atomicAdd(&hist[jl * 256 + bin], (uint32_t)__popc(peers));
              }
            }
          }
        }
      } else {
        tile_epilogue<D, NP>(es, acc, ea, ls, q, lane, et, sc, tok, valid, counting, p, b, j0, start, vstage_w);
      }
    }
    if (!DUMP) {
      // the warps' states go into the key ring: it is free once a warp has
      // seen the last tile's scores (every MMA and copy is done)
      tail_merge<D, NP>(es, reinterpret_cast<float*>(kst), acc, ls, ea, vstage, q, lane, et, p, b, j0, s,
                        t != ntiles);
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  const bool aborted = *abort_flag != 0;
  if (aborted) {
    if (threadIdx.x == 0) flag_status(p.status, SAGA_STATUS_TIMEOUT);
    if (warp == 0 && lane == 0) {
      // wait (bounded) for the last copy issued into each stage
      for (int t = max(0, issued - NSTAGE); t < issued; ++t) mbar_wait_drain(&full[t % NSTAGE], (t / NSTAGE) & 1);
    }
  }
  if (DHIST && p.hist_out != nullptr && warp >= 2) {
    const int et = threadIdx.x - 64;
    for (int i = et; i < p.G * 256; i += kEpiThreads) {
      const uint32_t c = hist[i];
      if (c) atomicAdd(&p.hist_out[((size_t)b * p.h_q + j0 + i / 256) * 256 + (i % 256)], c);
    }
  }
  __syncthreads();
  if (UMMA && warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ============================================================================ from-scores kernel
// Refresh steps: the scores were dumped before the exact threshold was known;
// compare and gather from them with the same per-warp epilogue.
template <int NP>
__device__ __forceinline__ void load_scores(float (&dst)[NP], const float* srow, long long ld, int G, int tok, int end) {
#pragma unroll
  for (int jl = 0; jl < NP; ++jl) dst[jl] = (jl < G && tok < end) ? __ldg(srow + (size_t)jl * ld + tok) : -INFINITY;
}

// Value staging of the compare/gather pass: 4 KB per warp list buffer at
// d = 128 (half the split kernel's), so that two of its CTAs share an SM.
template <int D, int NP>
__host__ __device__ constexpr int fs_vstage_warp_bytes() {
  return (D == 128 && NP <= 16) ? 4096 : vstage_warp_bytes<D, NP>();
}

template <int D, int NP>
struct FromScoresSmem {
  static constexpr int VST_OFF = ((int)sizeof(EpiShared<NP>) + 127) / 128 * 128;
  static constexpr int MRG_OFF = VST_OFF + 4 * 2 * fs_vstage_warp_bytes<D, NP>();
  static constexpr int BYTES = MRG_OFF + merge_floats<D, NP>() * 4;
};

template <int D, int NP>
__global__ void __launch_bounds__(kEpiThreads) saga_from_scores_kernel(const SplitParams p) {
  using SM = FromScoresSmem<D, NP>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  EpiShared<NP>& es = *reinterpret_cast<EpiShared<NP>*>(smem_raw);
  uint16_t* vstage = reinterpret_cast<uint16_t*>(smem_raw + SM::VST_OFF);
  float* mrg = reinterpret_cast<float*>(smem_raw + SM::MRG_OFF);
  const CtaCoord cc = cta_coord(p);
  const int s = cc.s, h = cc.h, b = cc.b;
  const int et = threadIdx.x, q = et >> 5, lane = et & 31;
  const int j0 = cc.j0;
  pdl_trigger();
  pdl_wait();
  const int L = device_seq_len(p.seq_len_dev, p.seq_len, p.l_cap, nullptr);
  int start, end;
  split_range(p.seq_len, p.nsplit, s, L, &start, &end);
  const int ntiles = (end - start + kTile - 1) / kTile;
  const bool counting = p.want_counts != 0;

  epi_setup<NP>(es, et, p, load_tau<NP>(et, p, b, j0, true));  // dumped scores are scaled: compare as they are
  constexpr int VSB = fs_vstage_warp_bytes<D, NP>();
  EpiArgs ea = epi_args<D, NP, VSB>(p, b, j0);
  ea.scale = 1.f;  // the dumped scores are scaled already
  uint16_t* vstage_w = vstage + (size_t)q * 2 * (VSB / 2);
  WarpAcc<D, NP> acc;
  acc.init();
  ListState ls{0, 0, -1, 0};
  const float* srow = p.scores_in + ((size_t)b * p.h_q + j0) * (size_t)p.ld_scores;
  __syncthreads();

  float nxt[NP];
  if (ntiles > 0) load_scores<NP>(nxt, srow, p.ld_scores, p.G, start + et, end);
  for (int t = 0; t < ntiles; ++t) {
    float sc[NP];
#pragma unroll
    for (int jl = 0; jl < NP; ++jl) sc[jl] = nxt[jl];
    if (t + 1 < ntiles) load_scores<NP>(nxt, srow, p.ld_scores, p.G, start + (t + 1) * kTile + et, end);
    const int tok = start + t * kTile + et;
    tile_epilogue<D, NP>(es, acc, ea, ls, q, lane, et, sc, tok, tok < end, counting, p, b, j0, start, vstage_w);
  }
  tail_merge<D, NP, VSB>(es, mrg, acc, ls, ea, vstage, q, lane, et, p, b, j0, s, false);
}

// ============================================================================ dense kernel
// Attention with every token kept (N covers the context) and one value head
// per key-head group (h_v <= h_k): a tile's value rows are contiguous, so
// they come in by TMA with its key rows, and each epilogue warp runs the
// softmax and the value sum of its 32 rows per tile (online, no lists).
// Warp roles as in the split kernel; the partials feed the same combine.
#ifndef SAGA_DENSE_SETS
#define SAGA_DENSE_SETS 2
#endif
constexpr int kDenseSetsSmallGroups = SAGA_DENSE_SETS;  // epilogue sets of the dense kernel at <= 4 heads

template <int D, int NP>
struct DenseSmem {
  static constexpr int NATOM = D / 64;
  static constexpr int KBYTES = kTile * D * 2;
  static constexpr int STAGE_BYTES = 2 * KBYTES;  // key tile (128-byte swizzle) + value tile (no swizzle)
  static constexpr int NPM = mma_n<NP>();
  static constexpr int NACC = acc_bufs<NP>();
  static constexpr int QPAD = ((NATOM * NPM * 128 + 1023) / 1024) * 1024;
  // epilogue sets: with 4 heads a set of four warps is issue-bound on the
  // value sums, so two sets take alternate tiles (8 epilogue warps)
  static constexpr int ESETS = NP <= 4 ? kDenseSetsSmallGroups : 1;
  static constexpr int THREADS = 64 + 128 * ESETS;
  static constexpr int PBUF_BYTES = 4 * ESETS * 32 * NP * 4;  // each epilogue warp's weights of a tile, [32][NP]
  static constexpr int FIXED = QPAD + PBUF_BYTES + (2 * 4 + 2 * NACC + 1) * 8 + 16 + 1024;
  static constexpr int NSTAGE_HALF = (kSmemHalf - FIXED) / STAGE_BYTES;
  static constexpr bool TWO = NSTAGE_HALF >= 3;  // two CTAs per SM with 3 stages each
  static constexpr int NSTAGE_FIT = (kSmemLimit - FIXED) / STAGE_BYTES;
  static constexpr int NSTAGE = TWO ? 3 : (NSTAGE_FIT < 4 ? NSTAGE_FIT : 4);
  static constexpr int CTAS_PER_SM = TWO ? 2 : 1;
  static constexpr int Q_OFF = NSTAGE * STAGE_BYTES;
  static constexpr int P_OFF = Q_OFF + QPAD;
  static constexpr int BAR_OFF = P_OFF + PBUF_BYTES;
  static constexpr int NBARS = 2 * NSTAGE + 2 * NACC + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static_assert(NSTAGE >= 2, "ring too shallow");
  static_assert(ALLOC <= kSmemLimit, "shared memory over the per-CTA limit");
  static_assert(!TWO || ALLOC <= kSmemHalf, "two CTAs per SM must fit in half the shared memory");
  static_assert(4 * ESETS * NP * (D + 2) * 4 <= NSTAGE * STAGE_BYTES, "merge buffer must fit in the ring");
};

// Key and value rows of tile t into its stage (128-row boxes, or 32-row
// boxes for the rows left in the split).
template <int NATOM, int NSTAGE, int STAGE_BYTES, int KBYTES>
__device__ __forceinline__ void issue_kv_tile(int t, int start, int end, int krow, int vrow, uint8_t* ring,
                                              uint64_t* full, const CUtensorMap* tkf, const CUtensorMap* tkp,
                                              const CUtensorMap* tvf, const CUtensorMap* tvp) {
  const int stage = t % NSTAGE;
  const int r0 = start + t * kTile;
  const int rows = min(kTile, end - r0);
  uint8_t* dst = ring + stage * STAGE_BYTES;
  if (rows == kTile) {
    mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
#pragma unroll
    for (int a = 0; a < NATOM; ++a) {
      tma_load_2d(dst + a * 16384, tkf, &full[stage], a * 64, krow + r0);
      tma_load_2d(dst + KBYTES + a * 16384, tvf, &full[stage], a * 64, vrow + r0);
    }
  } else {
    const int nsub = (rows + kUnit - 1) / kUnit;
    mbar_arrive_expect_tx(&full[stage], 2 * nsub * kUnit * 128 * NATOM);
    for (int i = 0; i < nsub; ++i)
#pragma unroll
      for (int a = 0; a < NATOM; ++a) {
        tma_load_2d(dst + a * 16384 + i * kUnit * 128, tkp, &full[stage], a * 64, krow + r0 + i * kUnit);
        tma_load_2d(dst + KBYTES + a * 16384 + i * kUnit * 128, tvp, &full[stage], a * 64, vrow + r0 + i * kUnit);
      }
  }
}

template <int D, int NP>
__global__ void __launch_bounds__(DenseSmem<D, NP>::THREADS, DenseSmem<D, NP>::CTAS_PER_SM)
    saga_dense_kernel(const __grid_constant__ CUtensorMap tk_full, const __grid_constant__ CUtensorMap tk_part,
                      const __grid_constant__ CUtensorMap tv_full, const __grid_constant__ CUtensorMap tv_part,
                      const SplitParams p) {
  using SM = DenseSmem<D, NP>;
  constexpr int NATOM = SM::NATOM;
  constexpr int NSTAGE = SM::NSTAGE;
  constexpr int STAGE_BYTES = SM::STAGE_BYTES;
  constexpr int KBYTES = SM::KBYTES;
  constexpr int NPM = SM::NPM;
  constexpr int NACC = SM::NACC;
  constexpr int ESETS = SM::ESETS;
  constexpr int NEPI = 128 * ESETS;  // epilogue threads
  constexpr int DPL = D / 32;
  constexpr uint32_t TMEM_COLS = NACC * NPM <= 32 ? 32u : NACC * NPM <= 64 ? 64u : NACC * NPM <= 128 ? 128u : 256u;
  constexpr uint32_t IDESC = umma_idesc_bf16(128, NPM);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* qsm = smem + SM::Q_OFF;
  float* pbuf = reinterpret_cast<float*>(smem + SM::P_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::BAR_OFF);
  uint64_t* empty = full + NSTAGE;
  uint64_t* accf = empty + NSTAGE;
  uint64_t* acce = accf + NACC;
  uint64_t* fin = acce + NACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::MISC_OFF + 4);

  const CtaCoord cc = cta_coord(p);
  const int s = cc.s, h = cc.h, b = cc.b;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = cc.j0;
  const int v_base = (int)(((long long)j0 * p.h_v) / p.h_q);
  const int krow = (b * p.h_k + h) * p.l_cap;       // first cache row of this (batch, key head)
  const int vrow = (b * p.h_v + v_base) * p.l_cap;  // ... and of its value head

  // ---------------------------------------------------------------- setup before the dependency wait
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1 + 4);  // the MMA's commit and the four epilogue warps
    }
    for (int i = 0; i < NACC; ++i) {
      mbar_init(&accf[i], 1);
      mbar_init(&acce[i], 4);
    }
    mbar_init(fin, 1);
    mbar_init_fence();
    tma_prefetch_desc(&tk_full);
    tma_prefetch_desc(&tk_part);
    tma_prefetch_desc(&tv_full);
    tma_prefetch_desc(&tv_part);
    int pst, pcap;
    split_cap_range(p.seq_len, p.nsplit, s, p.l_cap, &pst, &pcap);
    const long long ncta = (long long)gridDim.x * gridDim.y * gridDim.z;
    const int cap_rows = max(kTile, (int)(((48ll << 20) / ncta) / (2 * D * 2)) / kTile * kTile);
    const int pend = min(pcap, pst + cap_rows);
    for (int r = pst; r < pend; r += kTile) {
      const uint32_t bytes = (uint32_t)(min(kTile, pend - r) * D * 2);
      prefetch_l2_bulk(p.k_cache + ((size_t)krow + r) * D, bytes);
      prefetch_l2_bulk(p.v_cache + ((size_t)vrow + r) * D, bytes);
    }
  } else if (warp == 2) {
    const char* qg = reinterpret_cast<const char*>(p.q + ((size_t)b * p.h_q + j0) * D);
    for (int i = lane; i < p.G * D * 2 / 128; i += 32) prefetch_l2_line(qg + 128 * i);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();

  // ---------------------------------------------------------------- setup after it
  constexpr int QCH = NATOM * NPM * 8;
  constexpr int QV = (QCH + kEpiThreads - 1) / kEpiThreads;
  const int eth = threadIdx.x - 64;
  uint4 qv[QV];
  const bool qstage = warp >= 2 && warp < 6;  // the first epilogue set stages q
  if (qstage) {
#pragma unroll
    for (int k = 0; k < QV; ++k) {
      const int i = eth + k * kEpiThreads;
      const int n = (i / 8) % NPM, col = (i / (NPM * 8)) * 64 + (i % 8) * 8;
      qv[k] = make_uint4(0, 0, 0, 0);
      if (i < QCH && n < p.G) qv[k] = __ldg(reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.h_q + j0 + n) * D + col));
    }
  }
  const int L = device_seq_len(p.seq_len_dev, p.seq_len, p.l_cap, (s == 0 && h == 0 && b == 0) ? p.status : nullptr);
  int start, end;
  split_range(p.seq_len, p.nsplit, s, L, &start, &end);
  const int ntiles = (end - start + kTile - 1) / kTile;
  const bool owner = p.k_new != nullptr && start <= L - 1 && L - 1 < end;
  if (owner) append_new_rows<D>(p, b, h, j0, L - 1);
  int issued = 0;
  if (threadIdx.x == 0) {
    for (; issued < ntiles && issued < NSTAGE; ++issued) {
      if (owner && L - 1 < start + (issued + 1) * kTile) break;
      issue_kv_tile<NATOM, NSTAGE, STAGE_BYTES, KBYTES>(issued, start, end, krow, vrow, ring, full, &tk_full, &tk_part,
                                                        &tv_full, &tv_part);
    }
  }
  if (qstage) {
#pragma unroll
    for (int k = 0; k < QV; ++k) {
      const int i = eth + k * kEpiThreads;
      if (i < QCH) {
        const int a = i / (NPM * 8), n = (i / 8) % NPM, c = i % 8;
        *reinterpret_cast<uint4*>(qsm + a * NPM * 128 + n * 128 + ((c ^ (n & 7)) << 4)) = qv[k];
      }
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // ---------------------------------------------------------------- roles
  if (warp == 0) {
    if (lane == 0) {
      if (owner) fence_proxy_async_global();
      for (int t = issued; t < ntiles; ++t) {
        const int stage = t % NSTAGE, round = t / NSTAGE;
        if (round > 0 && !mbar_wait(&empty[stage], (round - 1) & 1, abort_flag)) break;
        issue_kv_tile<NATOM, NSTAGE, STAGE_BYTES, KBYTES>(t, start, end, krow, vrow, ring, full, &tk_full, &tk_part,
                                                          &tv_full, &tv_part);
        issued = t + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      for (int t = 0; t < ntiles; ++t) {
        const int stage = t % NSTAGE, round = t / NSTAGE;
        if (!mbar_wait(&full[stage], round & 1, abort_flag)) break;
        const int abuf = t % NACC;
        if (t >= NACC && !mbar_wait(&acce[abuf], ((t / NACC) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(ring + stage * STAGE_BYTES);
        const uint32_t b0 = smem_u32(qsm);
        const uint32_t d_tmem = tmem_base + abuf * NPM;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t aa = a0 + (k >> 2) * 16384 + (k & 3) * 32;
          const uint32_t bb = b0 + (k >> 2) * NPM * 128 + (k & 3) * 32;
          umma_bf16(d_tmem, umma_sdesc_sw128(aa), umma_sdesc_sw128(bb), IDESC, k > 0 ? 1u : 0u);
        }
        umma_commit(&empty[stage]);
        umma_commit(&accf[abuf]);
      }
      umma_commit(fin);
      if (!mbar_wait_drain(fin, 0)) *abort_flag = 1;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // set es of four warps takes tiles es, es + ESETS, ...; within a set the
    // warps own the TMEM lane quarters (warp mod 4)
    const int et = threadIdx.x - 64;
    const int ew = warp - 2;    // epilogue warp 0 .. 4 * ESETS - 1
    const int eset = ew >> 2;
    const int q = warp & 3;     // TMEM lane quarter: rows 32q .. 32q+31 of every tile
    const int erow = 32 * q + lane;
    const bool counting = p.want_counts != 0;
    float m[NP], lp[NP], o[NP][DPL];  // running max (warp-uniform), per-lane weight sums, columns of the lane
#pragma unroll
    for (int jl = 0; jl < NP; ++jl) {
      m[jl] = -INFINITY;
      lp[jl] = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) o[jl][e] = 0.f;
    }
    float* pw = pbuf + ew * 32 * NP;
    // the lane's columns of a value row: atom (lane*DPL)/64, byte offset within the 128-byte row
    const int vcol = ((lane * DPL) / 64) * 16384 + ((lane * DPL) % 64) * 2;
    for (int t = eset; t < ntiles; t += ESETS) {
      const int stage = t % NSTAGE;
      const int abuf = t % NACC;
      if (!__all_sync(0xffffffffu, mbar_wait(&accf[abuf], (t / NACC) & 1, abort_flag))) break;
      tc_fence_after();
      float sc[NP];
      {
        const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(abuf * NPM);
        if constexpr (NP >= 16) {
#pragma unroll
          for (int i = 0; i < NP / 16; ++i) tmem_ld16(taddr + 16 * i, sc + 16 * i);
        } else {
          float all[16];
          tmem_ld16(taddr, all);
#pragma unroll
          for (int i = 0; i < NP; ++i) sc[i] = all[i];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[abuf]);
      const int tok = start + t * kTile + erow;
      const bool valid = tok < end;
      // online softmax of the warp's 32 rows, per head
#pragma unroll
      for (int jl = 0; jl < NP; ++jl) {
        float pj = 0.f;
        if (jl < p.G) {
          const float x = sc[jl] * p.scale;
          const uint32_t kmax = __reduce_max_sync(0xffffffffu, valid ? float_key(x) : 0u);
          if (kmax != 0u) {  // warp-uniform
            const float tm = key_float(kmax);
            if (tm > m[jl]) {
              const float f = (m[jl] == -INFINITY) ? 0.f : __expf(m[jl] - tm);
              lp[jl] *= f;
#pragma unroll
              for (int e = 0; e < DPL; ++e) o[jl][e] *= f;
              m[jl] = tm;
            }
          }
          pj = valid ? __expf(x - m[jl]) : 0.f;
          if (counting && valid) p.idxbuf[((size_t)b * p.h_q + j0 + jl) * p.l_cap + tok] = tok;
        }
        lp[jl] += pj;
        sc[jl] = pj;
      }
#pragma unroll
      for (int j4 = 0; j4 < NP / 4; ++j4)
        *reinterpret_cast<float4*>(&pw[lane * NP + 4 * j4]) =
            make_float4(sc[4 * j4], sc[4 * j4 + 1], sc[4 * j4 + 2], sc[4 * j4 + 3]);
      // the value tile landed with the key tile (same stage barrier)
      mbar_wait(&full[stage], (t / NSTAGE) & 1, abort_flag);
      __syncwarp();
      const uint8_t* vt = ring + stage * STAGE_BYTES + KBYTES + (32 * q) * 128 + vcol;
      // rows past the split's end hold no loaded values (stale or outside
      // data): never read them, even with weight 0 (0 * NaN is NaN)
      const int nrows = min(32, max(0, end - (start + t * kTile + 32 * q)));
#pragma unroll 4
      for (int r = 0; r < nrows; ++r) {
        float w[NP];
#pragma unroll
        for (int j4 = 0; j4 < NP / 4; ++j4) {
          const float4 w4 = *reinterpret_cast<const float4*>(&pw[r * NP + 4 * j4]);
          w[4 * j4] = w4.x;
          w[4 * j4 + 1] = w4.y;
          w[4 * j4 + 2] = w4.z;
          w[4 * j4 + 3] = w4.w;
        }
        float v[DPL];
        load_bf16<DPL>(reinterpret_cast<const uint16_t*>(vt + r * 128), v);
#pragma unroll
        for (int jl = 0; jl < NP; ++jl)
          if (jl < p.G) {
#pragma unroll
            for (int e = 0; e < DPL; ++e) o[jl][e] = fmaf(w[jl], v[e], o[jl][e]);
          }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
    }
    // ---- merge the epilogue warps' states and write the split's partial
    constexpr int REG = NP * (D + 2);
    constexpr int NW = 4 * ESETS;
    float lw[NP];
#pragma unroll
    for (int jl = 0; jl < NP; ++jl) lw[jl] = warp_sum(lp[jl]);
    named_bar_sync(1, NEPI);  // every warp is done with the ring (value rows)
    float* mrg = reinterpret_cast<float*>(ring);
    float* mine = mrg + ew * REG;
    if (lane == 0) {
#pragma unroll
      for (int jl = 0; jl < NP; ++jl) {
        mine[jl] = m[jl];
        mine[NP + jl] = lw[jl];
      }
    }
#pragma unroll
    for (int jl = 0; jl < NP; ++jl)
#pragma unroll
      for (int e = 0; e < DPL; ++e) mine[2 * NP + jl * D + lane * DPL + e] = o[jl][e];
    named_bar_sync(1, NEPI);
    const size_t row0 = (size_t)b * p.h_q + j0;
    for (int idx = et; idx < p.G * (D / 4); idx += NEPI) {
      const int jl = idx / (D / 4), c4 = idx % (D / 4);
      float m4[NW], M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        m4[w] = mrg[w * REG + jl];
        M = fmaxf(M, m4[w]);
      }
      float4 acc4 = make_float4(0.f, 0.f, 0.f, 0.f);
      float lsum = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float f = (m4[w] == -INFINITY) ? 0.f : __expf(m4[w] - M);
        const float4 v = *reinterpret_cast<const float4*>(&mrg[w * REG + 2 * NP + jl * D + c4 * 4]);
        acc4.x = fmaf(f, v.x, acc4.x);
        acc4.y = fmaf(f, v.y, acc4.y);
        acc4.z = fmaf(f, v.z, acc4.z);
        acc4.w = fmaf(f, v.w, acc4.w);
        lsum = fmaf(f, mrg[w * REG + NP + jl], lsum);
      }
      *reinterpret_cast<float4*>(&p.part_o[((row0 + jl) * p.s_cap + s) * D + c4 * 4]) = acc4;
      if (c4 == 0) {
        p.part_m[(row0 + jl) * p.s_cap + s] = M;
        p.part_l[(row0 + jl) * p.s_cap + s] = lsum;
        p.part_cnt[(row0 + jl) * p.s_cap + s] = end - start;
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (*abort_flag != 0) {
    if (threadIdx.x == 0) flag_status(p.status, SAGA_STATUS_TIMEOUT);
    if (warp == 0 && lane == 0)
      for (int t = max(0, issued - NSTAGE); t < issued; ++t) mbar_wait_drain(&full[t % NSTAGE], (t / NSTAGE) & 1);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ============================================================================ combine kernel
// O[b, j] = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s over the splits of
// row (b, j); zero when nothing was kept.  Also the kept counts and the
// ascending index list (concatenation of the per-split lists in split order).

// Grid: (B*h_q rows, D/32 column chunks).  Warp w of a CTA takes the splits
// [w*U, w*U + U) of each round of NW*U (one round for up to 192 splits):
// lane u loads the (m, l) of split u, the warp reduces them, and every lane
// loads the partial o of all U splits in its column (32*chunk + lane, so
// each load is one coalesced 128-byte segment), all in flight at once,
// weighting them with the shuffled factors.  The eight warps' states are
// merged at the end in a fixed order (deterministic).
// At most 64 registers a thread (16K for the CTA): with the 48K of a d = 128
// split CTA that fills the SM's register file, so a combine CTA and a split
// CTA of the next call share an SM - the split CTAs are resident before
// their dependency wait ends.
constexpr int kCombineThreads = 256;

template <int D>
__global__ void __launch_bounds__(kCombineThreads, 4) saga_combine_kernel(const CombineParams p) {
  constexpr int NW = kCombineThreads / 32;
  constexpr int U = 24;
  __shared__ float wm[NW], wden[NW];
  __shared__ float wacc[NW][32];
  __shared__ int cnt_scan[kCombineThreads];
  const int row = blockIdx.x, chunk = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();
  const int S = p.nsplit;
  const float* pm = p.part_m + (size_t)row * p.s_cap;
  const float* pl = p.part_l + (size_t)row * p.s_cap;
  const float* po = p.part_o + (size_t)row * p.s_cap * D + chunk * 32 + lane;

  float m_run = -INFINITY, den = 0.f, acc = 0.f;
  for (int s0 = warp * U; s0 < S; s0 += U * NW) {
    const int su = s0 + lane;
    const bool own = lane < U && su < S;
    const float mu = own ? pm[su] : -INFINITY;
    const float lu = own ? pl[su] : 0.f;
    float v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) v[u] = s0 + u < S ? po[(size_t)(s0 + u) * D] : 0.f;
    const float mb = warp_max(mu);
    if (mb > m_run) {  // warp-uniform
      const float f = (m_run == -INFINITY) ? 0.f : __expf(m_run - mb);
      den *= f;
      acc *= f;
      m_run = mb;
    }
    const float fu = (mu == -INFINITY) ? 0.f : __expf(mu - m_run);
    den += warp_sum(fu * lu);
#pragma unroll
    for (int u = 0; u < U; ++u) acc = fmaf(__shfl_sync(0xffffffffu, fu, u), v[u], acc);
  }
  wacc[warp][lane] = acc;
  if (lane == 0) {
    wm[warp] = m_run;
    wden[warp] = den;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, wm[w]);
    float num = 0.f, dd = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float f = (wm[w] == -INFINITY) ? 0.f : __expf(wm[w] - M);
      num = fmaf(f, wacc[w][threadIdx.x], num);
      dd = fmaf(f, wden[w], dd);
    }
    const float o = (M == -INFINITY || dd <= 0.f) ? 0.f : num / dd;
    const size_t oi = (size_t)row * D + chunk * 32 + threadIdx.x;
    if (p.out_bf16) {
      reinterpret_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(o);
    } else {
      reinterpret_cast<float*>(p.out)[oi] = o;
    }
  }
  if (chunk != 0) return;
  if (p.sel_count == nullptr) return;
  // kept counts and index lists
  const int* pc = p.part_cnt + (size_t)row * p.s_cap;
  int total = 0;
  for (int base = 0; base < S; base += kCombineThreads) {
    const int s = base + threadIdx.x;
    const int c = s < S ? pc[s] : 0;
    cnt_scan[threadIdx.x] = c;
    __syncthreads();
    for (int off = 1; off < kCombineThreads; off <<= 1) {
      const int v = threadIdx.x >= off ? cnt_scan[threadIdx.x - off] : 0;
      __syncthreads();
      cnt_scan[threadIdx.x] += v;
      __syncthreads();
    }
    const int incl = cnt_scan[threadIdx.x];
    const int chunk_total = cnt_scan[kCombineThreads - 1];
    __syncthreads();
    if (p.sel_idx != nullptr && s < S) cnt_scan[threadIdx.x] = total + incl - c;  // exclusive offset
    __syncthreads();
    if (p.sel_idx != nullptr) {
      const int L = device_seq_len(p.seq_len_dev, p.seq_len, p.l_cap, nullptr);
      const int nloc = min(kCombineThreads, S - base);
      for (int k = warp; k < nloc; k += NW) {
        const int ss = base + k;
        int st, en;
        split_range(p.seq_len, S, ss, L, &st, &en);
        const int cnt = pc[ss];
        const int off = cnt_scan[k];
        const int* src = p.idxbuf + (size_t)row * p.l_cap + st;
        int* dst = p.sel_idx + (size_t)row * p.l_cap + off;
        for (int i = lane; i < cnt; i += 32) dst[i] = src[i];
      }
    }
    total += chunk_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) p.sel_count[row] = total;
}

// ============================================================================ radix select
// Exact N-th largest per row: MSB-first 8-bit digits of the order-preserving
// key; candidates of the current digit bin are moved to shared memory once
// they fit, and the remaining digits are resolved there.
// Adds one to hist[bin] for every lane with `valid` (lanes with the same bin
// are grouped first, so each bin takes one shared-memory atomic per warp).
// Called with warp-uniform control flow; a warp with no valid lane skips the
// grouping.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool valid) {
  if (!__any_sync(0xffffffffu, valid)) return;
  const uint32_t key = valid ? bin : 0xFFFFFFFFu;
  const uint32_t peers = __match_any_sync(0xffffffffu, key);
  if (valid && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

// Appends k to cand when take (warp-aggregated: one shared atomic per warp);
// *ncand counts every taken key, also those past kSelectCap.  Full warp.
__device__ __forceinline__ void cand_add(uint32_t* cand, int* ncand, uint32_t k, bool take) {
  const uint32_t m = __ballot_sync(0xffffffffu, take);
  if (m == 0u) return;
  const int lane = threadIdx.x & 31, first = __ffs(m) - 1;
  int base = 0;
  if (lane == first) base = atomicAdd(ncand, __popc(m));
  base = __shfl_sync(0xffffffffu, base, first);
  const int pos = base + __popc(m & ((1u << lane) - 1u));
  if (take && pos < kSelectCap) cand[pos] = k;
}

// Top-byte bin of row r's stale threshold, from which the top-digit pass also
// keeps candidates (the N-th largest mostly stays in its bin from one refresh
// to the next); 256 = none: not asked, or a threshold that is not a positive
// finite number (from 0 down the kept keys would take in every positive
// score, as at a session's first refresh, whose thresholds start at 0).
__device__ __forceinline__ uint32_t spec_floor(const SelectParams& p, int r) {
  if (p.spec == 0) return 256u;
  const float t = p.tau[r];
  return isfinite(t) && t > 0.f ? float_key(t) >> 24 : 256u;
}

// Float4 loads each thread keeps in flight in the row scans.
constexpr int kScanUnroll = 4;

// Calls f(key, valid) for every element of row[0, L) with warp-uniform trip
// counts (so f may use full-warp primitives).  row is 16-byte aligned.
template <typename F>
__device__ __forceinline__ void scan_row(const float* row, int L, F&& f) {
  const int nvec = L >> 2;
  const int nvec_pad = (nvec + 31) & ~31;
  const float4* row4 = reinterpret_cast<const float4*>(row);
  for (int i0 = threadIdx.x; i0 < nvec_pad; i0 += kSelectThreads * kScanUnroll) {
    float4 v[kScanUnroll];
#pragma unroll
    for (int u = 0; u < kScanUnroll; ++u) {
      const int i = i0 + u * kSelectThreads;
      v[u] = i < nvec ? __ldg(row4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kScanUnroll; ++u) {
      const int i = i0 + u * kSelectThreads;
      if (i < nvec_pad) {  // warp-uniform (i is 32-aligned within a warp)
        const bool inb = i < nvec;
        f(float_key(v[u].x), inb);
        f(float_key(v[u].y), inb);
        f(float_key(v[u].z), inb);
        f(float_key(v[u].w), inb);
      }
    }
  }
  if (threadIdx.x < 32) {
    const int i = 4 * nvec + threadIdx.x;
    const bool inb = i < L;
    f(inb ? float_key(row[i]) : 0u, inb);
  }
}

// Finds the digit bin holding the rank-th largest (rank 1-based), given a
// 256-bin histogram; returns bin, rank within the bin, and the bin count.
__device__ void find_bin(const uint32_t* hist, uint32_t rank, uint32_t* out_bin, uint32_t* out_rank,
                         uint32_t* out_cnt) {
  // warp 0: lane l owns bins 255-8l ... 248-8l (descending)
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    uint32_t loc = 0;
    for (int i = 0; i < 8; ++i) loc += hist[255 - 8 * lane - i];
    uint32_t incl = loc;
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - loc;
    if (rank > excl && rank <= incl) {
      uint32_t above = excl;
      for (int i = 0; i < 8; ++i) {
        const int bin = 255 - 8 * lane - i;
        const uint32_t c = hist[bin];
        if (rank <= above + c) {
          *out_bin = (uint32_t)bin;
          *out_rank = rank - above;
          *out_cnt = c;
          break;
        }
        above += c;
      }
    }
  }
}

__global__ void __launch_bounds__(kSelectThreads) atopn_select_kernel(const SelectParams p) {
  extern __shared__ uint32_t cand[];  // kSelectCap keys
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_bin, s_rank, s_cnt;
  __shared__ int ncand;
  const int r = blockIdx.x;
  pdl_trigger();
  pdl_wait();
  int L = p.row_len;
  if (p.seq_len_dev != nullptr) L = device_seq_len(p.seq_len_dev, p.row_len, p.l_cap, nullptr);
  if (p.n_top >= L) {
    if (threadIdx.x == 0) p.tau[r] = -INFINITY;
    return;
  }
  const float* row = p.scores + (size_t)r * p.ld;
  const uint32_t fl = spec_floor(p, r);  // read before this CTA writes tau[r]

  // given top-digit counts may hold only the bins from some floor up (the
  // score dump counts from just below the stale threshold): they serve when
  // their bins hold at least N scores, else the row is counted here
  __shared__ uint32_t counted;
  if (threadIdx.x == 0) {
    ncand = 0;
    s_bin = 0;
    s_rank = 1;
    s_cnt = 0;
    counted = 0u;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 256; i += kSelectThreads) {
    hist[i] = p.hist != nullptr ? p.hist[(size_t)r * 256 + i] : 0u;
    if (hist[i] != 0u) atomicAdd(&counted, hist[i]);
  }
  __syncthreads();
  bool spec = false;  // uniform: the top-digit pass also kept the keys from bin fl up
  if (p.hist == nullptr || counted < (uint32_t)p.n_top) {  // top digit: a histogram of the whole row
    for (int i = threadIdx.x; i < 256; i += kSelectThreads) hist[i] = 0u;
    __syncthreads();
    if (fl < 256u) {
      spec = true;
      scan_row(row, L, [&](uint32_t k, bool ok) {
        hist_add(hist, k >> 24, ok);
        cand_add(cand, &ncand, k, ok && (k >> 24) >= fl);
      });
    } else {
      scan_row(row, L, [&](uint32_t k, bool ok) { hist_add(hist, k >> 24, ok); });
    }
    __syncthreads();
  }
  find_bin(hist, (uint32_t)p.n_top, &s_bin, &s_rank, &s_cnt);
  __syncthreads();
  uint32_t prefix = s_bin << 24, mask = 0xFF000000u, rank = s_rank, cnt = s_cnt;
  // the kept keys hold every key of the N-th largest's bin when that bin is fl
  // or above and none was dropped; else they are discarded and collected below
  bool in_smem = spec && s_bin >= fl && ncand <= kSelectCap;
  __syncthreads();  // every thread has read ncand
  if (!in_smem && threadIdx.x == 0) ncand = 0;
  __syncthreads();
  for (int shift = 16; shift >= 0; shift -= 8) {
    if (!in_smem && cnt <= (uint32_t)kSelectCap) {
      scan_row(row, L, [&](uint32_t k, bool ok) {
        if (ok && (k & mask) == prefix) {
          const int pos = atomicAdd(&ncand, 1);
          if (pos < kSelectCap) cand[pos] = k;
        }
      });
      in_smem = true;
    }
    for (int i = threadIdx.x; i < 256; i += kSelectThreads) hist[i] = 0u;
    __syncthreads();
    if (in_smem) {
      const int n = min(ncand, kSelectCap);
      for (int i = threadIdx.x; i < ((n + 31) & ~31); i += kSelectThreads) {
        const bool ok = i < n && (cand[i] & mask) == prefix;
        hist_add(hist, ok ? (cand[i] >> shift) & 255u : 0u, ok);
      }
    } else {
      scan_row(row, L, [&](uint32_t k, bool ok) {
        const bool m = ok && (k & mask) == prefix;
        hist_add(hist, m ? (k >> shift) & 255u : 0u, m);
      });
    }
    __syncthreads();
    find_bin(hist, rank, &s_bin, &s_rank, &s_cnt);
    __syncthreads();
    prefix |= s_bin << shift;
    mask |= 0xFFu << shift;
    rank = s_rank;
    cnt = s_cnt;
    __syncthreads();
  }
  if (threadIdx.x == 0) p.tau[r] = key_float(prefix);
}

// ---------------------------------------------------------------------------- cluster select
// Few long rows: the row in chunks over the CTAs of one thread-block cluster
// (atopn_cluster_select_kernel below).

// Calls f(key, valid) for the elements [begin, end) of row (begin a multiple
// of 4, row 16-byte aligned) with warp-uniform trip counts.
template <typename F>
__device__ __forceinline__ void scan_range(const float* row, int begin, int end, F&& f) {
  const int v0 = begin >> 2, v1 = end >> 2;  // whole float4 vectors
  const int nvec = max(0, v1 - v0);
  const int nvec_pad = (nvec + 31) & ~31;
  const float4* row4 = reinterpret_cast<const float4*>(row);
  const int nt = blockDim.x;
  for (int i0 = threadIdx.x; i0 < nvec_pad; i0 += nt * kScanUnroll) {
    float4 v[kScanUnroll];
#pragma unroll
    for (int u = 0; u < kScanUnroll; ++u) {
      const int i = i0 + u * nt;
      v[u] = i < nvec ? __ldg(row4 + v0 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kScanUnroll; ++u) {
      const int i = i0 + u * nt;
      if (i < nvec_pad) {  // warp-uniform (i is 32-aligned within a warp)
        const bool inb = i < nvec;
        f(float_key(v[u].x), inb);
        f(float_key(v[u].y), inb);
        f(float_key(v[u].z), inb);
        f(float_key(v[u].w), inb);
      }
    }
  }
  if (threadIdx.x < 32) {  // the last 0..3 elements
    const int i = 4 * max(v1, v0) + threadIdx.x;
    const bool inb = i < end && i >= begin;
    f(inb ? float_key(row[i]) : 0u, inb);
  }
}

__device__ __forceinline__ void sel_chunk(int L, int part, int P, int* b, int* e) {
  const int chunk = (((L + P - 1) / P) + 3) & ~3;
  *b = min(L, part * chunk);
  *e = min(L, *b + chunk);
}

// Exact N-th largest of a few long rows: one thread-block cluster per row,
// each CTA scanning a contiguous chunk.  Per 8-bit digit (MSB first) every
// CTA histograms the keys of its chunk that match the digits found so far;
// after a cluster barrier each CTA adds the cluster's histograms over
// distributed shared memory (so every CTA holds the same sums and takes the
// same decision) and finds the digit's bin.  Once the keys matching the
// prefix fit, each CTA keeps its own in shared memory and the remaining
// digits are resolved over those.  Given top-digit counts (from the score
// dump) are used when their bins hold N scores.  On refresh steps the
// top-digit pass also keeps the keys from the stale threshold's bin up, which
// saves the collection pass when the N-th largest stays in or above that bin.
// Cluster barriers are hardware barriers every CTA reaches on every path.
constexpr int kSelCluster = 8;          // CTAs per row
constexpr int kSelClusterThreads = 512;

__global__ void __launch_bounds__(kSelClusterThreads) atopn_cluster_select_kernel(const SelectParams p) {
  extern __shared__ uint32_t ccand[];  // this CTA's candidates (kSelectCap keys)
  __shared__ uint32_t hist[256], tot[256];
  __shared__ uint32_t s_bin, s_rank, s_cnt, counted;
  __shared__ int ncand;
  const int c = blockIdx.x, r = blockIdx.y;  // rank in the cluster, row
  pdl_trigger();
  pdl_wait();
  int L = p.row_len;
  if (p.seq_len_dev != nullptr) L = device_seq_len(p.seq_len_dev, p.row_len, p.l_cap, nullptr);
  if (p.n_top >= L) {  // uniform over the cluster: no CTA reaches a cluster barrier
    if (c == 0 && threadIdx.x == 0) p.tau[r] = -INFINITY;
    return;
  }
  const float* row = p.scores + (size_t)r * p.ld;
  // read before the first cluster barrier, so before CTA 0 can write tau[r]
  const uint32_t fl = spec_floor(p, r);
  int beg, end;
  sel_chunk(L, c, kSelCluster, &beg, &end);
  // adds the cluster's histograms into tot (every CTA), then finds the bin of `rank`
  auto cluster_bin = [&](uint32_t rank) {
    __syncthreads();
    cluster_sync_all();
    for (int i = threadIdx.x; i < 256; i += kSelClusterThreads) {
      uint32_t sum = 0u;
#pragma unroll
      for (int cc = 0; cc < kSelCluster; ++cc) sum += ld_dsmem_u32(&hist[i], cc);
      tot[i] = sum;
    }
    cluster_sync_all();  // every CTA has read every histogram before any is cleared
    if (threadIdx.x == 0) {
      s_bin = 0;
      s_rank = 1;
      s_cnt = 0;
    }
    __syncthreads();
    find_bin(tot, rank, &s_bin, &s_rank, &s_cnt);
    __syncthreads();
  };
  if (threadIdx.x == 0) {
    ncand = 0;
    counted = 0u;
  }
  __syncthreads();
  // top digit: the given counts when their bins hold N scores, else this
  // CTA's chunk counted and the cluster's counts summed
  for (int i = threadIdx.x; i < 256; i += kSelClusterThreads) {
    tot[i] = p.hist != nullptr ? p.hist[(size_t)r * 256 + i] : 0u;
    if (tot[i] != 0u) atomicAdd(&counted, tot[i]);
  }
  __syncthreads();
  bool spec = false;  // uniform: the top-digit pass also kept this chunk's keys from bin fl up
  if (p.hist == nullptr || counted < (uint32_t)p.n_top) {  // uniform: every CTA read the same counts
    for (int i = threadIdx.x; i < 256; i += kSelClusterThreads) hist[i] = 0u;
    __syncthreads();
    if (fl < 256u) {
      spec = true;
      scan_range(row, beg, end, [&](uint32_t k, bool ok) {
        hist_add(hist, k >> 24, ok);
        cand_add(ccand, &ncand, k, ok && (k >> 24) >= fl);
      });
    } else {
      scan_range(row, beg, end, [&](uint32_t k, bool ok) { hist_add(hist, k >> 24, ok); });
    }
    cluster_bin((uint32_t)p.n_top);
  } else {
    if (threadIdx.x == 0) {
      s_bin = 0;
      s_rank = 1;
      s_cnt = 0;
    }
    __syncthreads();
    find_bin(tot, (uint32_t)p.n_top, &s_bin, &s_rank, &s_cnt);
    __syncthreads();
  }
  uint32_t prefix = s_bin << 24, mask = 0xFF000000u, rank = s_rank, cnt = s_cnt;
  // this CTA's kept keys hold every key of its chunk in the N-th largest's bin
  // when that bin is fl or above and none was dropped (decided per CTA: the
  // cluster barriers below do not depend on it)
  bool in_smem = spec && s_bin >= fl && ncand <= kSelectCap;
  __syncthreads();  // every thread has read ncand
  if (!in_smem && threadIdx.x == 0) ncand = 0;
  __syncthreads();
  for (int shift = 16; shift >= 0; shift -= 8) {
    if (!in_smem && cnt <= (uint32_t)kSelectCap) {  // this CTA's matches are at most the cluster's cnt
      scan_range(row, beg, end, [&](uint32_t k, bool ok) {
        if (ok && (k & mask) == prefix) {
          const int pos = atomicAdd(&ncand, 1);
          if (pos < kSelectCap) ccand[pos] = k;
        }
      });
      in_smem = true;
    }
    for (int i = threadIdx.x; i < 256; i += kSelClusterThreads) hist[i] = 0u;
    __syncthreads();
    if (in_smem) {
      const int n = min(ncand, kSelectCap);
      for (int i = threadIdx.x; i < ((n + 31) & ~31); i += kSelClusterThreads) {
        const bool ok = i < n && (ccand[i] & mask) == prefix;
        hist_add(hist, ok ? (ccand[i] >> shift) & 255u : 0u, ok);
      }
    } else {
      scan_range(row, beg, end, [&](uint32_t k, bool ok) {
        const bool m = ok && (k & mask) == prefix;
        hist_add(hist, m ? (k >> shift) & 255u : 0u, m);
      });
    }
    cluster_bin(rank);
    prefix |= s_bin << shift;
    mask |= 0xFFu << shift;
    rank = s_rank;
    cnt = s_cnt;
    __syncthreads();
  }
  if (c == 0 && threadIdx.x == 0) p.tau[r] = key_float(prefix);
}

// ============================================================================ append + fill
__global__ void saga_append_kernel(const AppendParams p) {
  const int chunks_row = p.d / 8;  // 16-byte chunks per row
  const int nk = p.batch * p.h_k * chunks_row, nv = p.batch * p.h_v * chunks_row;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  pdl_trigger();
  pdl_wait();
  if (i >= nk + nv) return;
  int pos = p.pos;
  if (p.seq_len_dev != nullptr) pos = device_seq_len(p.seq_len_dev, p.pos + 1, p.l_cap, i == 0 ? p.status : nullptr) - 1;
  if (i < nk) {
    const int row = i / chunks_row, c = i % chunks_row;  // row = b*h_k + h
    const uint4 v = reinterpret_cast<const uint4*>(p.k_new)[i];
    reinterpret_cast<uint4*>(p.k_cache + ((size_t)row * p.l_cap + pos) * p.d)[c] = v;
  } else {
    const int j = i - nk;
    const int row = j / chunks_row, c = j % chunks_row;
    const uint4 v = reinterpret_cast<const uint4*>(p.v_new)[j];
    reinterpret_cast<uint4*>(p.v_cache + ((size_t)row * p.l_cap + pos) * p.d)[c] = v;
  }
}

__global__ void saga_fill_kernel(float* dst, float v, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  pdl_trigger();
  pdl_wait();
  if (i < n) dst[i] = v;
}

// ============================================================================ QKV projection
// Eq. 1 for the new token: q = x W_Q, k = x W_K, v = x W_V with h_k key
// heads and h_v value heads (SAGA: fewer key rows to stream), the key and
// value rows written straight into the caches at the new position (the
// append of the decode step).  Both kernels stream the weight matrix once;
// the weights, which no earlier kernel writes, are requested before the
// dependency wait so their stream overlaps the tail of the preceding kernel.
//
// Batch 1 (a matrix-vector product, 2 flops per weight): CUDA cores.  One
// warp per output column; each lane holds 16-byte pieces of the column's
// weight row in registers (the whole row of a 2048-wide model in flight at
// once) and multiplies them with x staged in shared memory; the warp sums the
// lanes' partial dot products.
constexpr int kQkvWarps = 8;                // output columns per CTA
constexpr int kQkvChunk = 2048;             // x elements per row staged per pass
constexpr int kQkvPieces = kQkvChunk / 256; // 16-byte weight pieces per lane per pass

// The new token's position: the host value, or seq_len - 1 read on the device.
__device__ __forceinline__ int qkv_position(const QkvParams& p) {
  return p.seq_len_dev != nullptr ? device_seq_len(p.seq_len_dev, p.pos + 1, p.l_cap, nullptr) - 1 : p.pos;
}

// Output column n of batch row b: the query, or row pos of a key or value head.
__device__ __forceinline__ void qkv_store(const QkvParams& p, int n, int b, int pos, float val) {
  const int qcols = p.h_q * p.d, kcols = p.h_k * p.d;
  const __nv_bfloat16 v = __float2bfloat16_rn(val);
  uint16_t bits;
  memcpy(&bits, &v, 2);
  if (n < qcols) {
    p.q[(size_t)b * qcols + n] = bits;
  } else if (n < qcols + kcols) {
    const int h = (n - qcols) / p.d, c = (n - qcols) % p.d;
    p.k_cache[(((size_t)b * p.h_k + h) * p.l_cap + pos) * p.d + c] = bits;
  } else {
    const int u = (n - qcols - kcols) / p.d, c = (n - qcols - kcols) % p.d;
    p.v_cache[(((size_t)b * p.h_v + u) * p.l_cap + pos) * p.d + c] = bits;
  }
}

template <int NB>
__global__ void __launch_bounds__(kQkvWarps * 32, NB == 1 ? 4 : 2) saga_qkv_kernel(const QkvParams p) {
  extern __shared__ __align__(16) uint16_t xs[];  // [NB][kQkvChunk]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * kQkvWarps + warp;
  const bool live = n < p.n_cols;
  const uint16_t* wrow = p.w + (size_t)(live ? n : 0) * p.hidden;
  uint4 wv[kQkvPieces];
  auto load_pass = [&](int k0, int kn) {
#pragma unroll
    for (int i = 0; i < kQkvPieces; ++i) {
      const int c = lane + 32 * i;  // piece index: elements 8c .. 8c + 7 of the pass
      wv[i] = live && c * 8 < kn ? __ldg(reinterpret_cast<const uint4*>(wrow + k0) + c) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  load_pass(0, min(kQkvChunk, p.hidden));
  if (live)  // later passes of a wider model: into L2 meanwhile
    for (int off = kQkvChunk * 2 + lane * 128; off < p.hidden * 2; off += 32 * 128)
      prefetch_l2_line(reinterpret_cast<const char*>(wrow) + off);
  pdl_trigger();
  pdl_wait();
  float acc[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[b] = 0.f;
  for (int k0 = 0; k0 < p.hidden; k0 += kQkvChunk) {
    const int kn = min(kQkvChunk, p.hidden - k0);
    if (k0 > 0) load_pass(k0, kn);
    __syncthreads();  // the previous pass is done with xs
    for (int i = threadIdx.x; i < NB * (kn / 8); i += blockDim.x) {
      const int b = i / (kn / 8), c = i % (kn / 8);
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (b < p.batch) v = __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)b * p.hidden + k0) + c);
      *reinterpret_cast<uint4*>(xs + b * kQkvChunk + c * 8) = v;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kQkvPieces; ++i) {
      const int c = lane + 32 * i;
      if (c * 8 >= kn) break;
      const float w0 = bf16_lo(wv[i].x), w1 = bf16_hi(wv[i].x), w2 = bf16_lo(wv[i].y), w3 = bf16_hi(wv[i].y);
      const float w4 = bf16_lo(wv[i].z), w5 = bf16_hi(wv[i].z), w6 = bf16_lo(wv[i].w), w7 = bf16_hi(wv[i].w);
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const uint4 xv = *reinterpret_cast<const uint4*>(xs + b * kQkvChunk + c * 8);
        float a = acc[b];
        a = fmaf(w0, bf16_lo(xv.x), a);
        a = fmaf(w1, bf16_hi(xv.x), a);
        a = fmaf(w2, bf16_lo(xv.y), a);
        a = fmaf(w3, bf16_hi(xv.y), a);
        a = fmaf(w4, bf16_lo(xv.z), a);
        a = fmaf(w5, bf16_hi(xv.z), a);
        a = fmaf(w6, bf16_lo(xv.w), a);
        a = fmaf(w7, bf16_hi(xv.w), a);
        acc[b] = a;
      }
    }
  }
  if (!live) return;
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[b] = warp_sum(acc[b]);
  // lane b writes batch row b of column n
  float mine = 0.f;
#pragma unroll
  for (int b = 0; b < NB; ++b)
    if (lane == b) mine = acc[b];
  if (lane < p.batch && lane < NB) qkv_store(p, n, lane, qkv_position(p), mine);
}

// Batch 2 .. 16 (up to 32 flops per weight byte pair: too many for CUDA cores
// to keep up with the weight stream): tcgen05.  The weight matrix is the A
// operand (M = 128 output columns per tile, K-major: row n of w_qkv), x the B
// operand (N = 16 batch rows, zero-padded); D[n][b] accumulates in TMEM.  The
// hidden dimension is split `splits` (<= 8) ways so that about one CTA per SM
// streams a share of the weights through a TMA ring; the splits of a tile form
// one thread-block cluster, each leaves its fp32 partial tile in its shared
// memory, and after a cluster barrier CTA r adds the partials of batch rows
// r, r + splits, ... in split order over distributed shared memory (the sum
// does not depend on timing) and writes the bf16 outputs.
constexpr int kQkvMmaThreads = 128;

__global__ void __launch_bounds__(kQkvMmaThreads)
    saga_qkv_mma_kernel(const __grid_constant__ CUtensorMap tw, const QkvParams p) {
  constexpr uint32_t IDESC = umma_idesc_bf16(kQkvTileM, kQkvN);
  constexpr uint32_t TMEM_COLS = 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem + p.stages * kQkvABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + qkv_mma_bar_offset(p.stages, p.kbs_max));
  uint64_t* empty = full + 8;
  uint64_t* accf = empty + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, tile = blockIdx.y;
  const int kb0 = (int)((long long)split * p.kb_total / p.splits);
  const int nkb = (int)((long long)(split + 1) * p.kb_total / p.splits) - kb0;  // >= 1: splits <= kb_total
  const int m0 = tile * kQkvTileM;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(accf, 1);
    mbar_init_fence();
    tma_prefetch_desc(&tw);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  int issued = 0;
  if (threadIdx.x == 0) {  // the first ring's worth of weight tiles, before the dependency wait
    const int first = min(nkb, p.stages);
    for (int i = 0; i < first; ++i) {
      mbar_arrive_expect_tx(&full[i], kQkvABytes);
      tma_load_2d(smem + i * kQkvABytes, &tw, &full[i], (kb0 + i) * kQkvTileK, m0);
    }
    issued = first;
  }
  pdl_trigger();
  pdl_wait();
  // x rows of this split's k-blocks into the 128-byte swizzle layout (16-byte
  // chunk c of row b at chunk position c ^ (b mod 8)); rows past the batch and
  // elements past hidden are zero.  Thread t owns chunk c = t mod 8 of row
  // b = t / 8 in every k-block; eight k-blocks' loads are in flight at once.
  static_assert(kQkvMmaThreads == kQkvN * 8, "one thread per 16-byte chunk of a k-block's x tile");
  {
    const int c = threadIdx.x & 7, b = threadIdx.x >> 3;
    const bool row_live = b < p.batch;
    const uint16_t* xrow = p.x + (size_t)(row_live ? b : 0) * p.hidden;
    uint8_t* xdst = xs + b * 128 + ((c ^ (b & 7)) << 4);
    for (int kq = 0; kq < nkb; kq += 8) {
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int k = (kb0 + kq + j) * kQkvTileK + c * 8;
        v[j] = make_uint4(0u, 0u, 0u, 0u);
        if (row_live && kq + j < nkb && k < p.hidden) v[j] = __ldg(reinterpret_cast<const uint4*>(xrow + k));
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (kq + j < nkb) *reinterpret_cast<uint4*>(xdst + (kq + j) * kQkvBBytes) = v[j];
    }
  }
  fence_proxy_async_shared();  // the generic-proxy writes above, seen by the tensor core
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = issued; kb < nkb; ++kb) {
        const int st = kb % p.stages, round = kb / p.stages;
        if (!mbar_wait(&empty[st], (round - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&full[st], kQkvABytes);
        tma_load_2d(smem + st * kQkvABytes, &tw, &full[st], (kb0 + kb) * kQkvTileK, m0);
        issued = kb + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      for (int kb = 0; kb < nkb; ++kb) {
        const int st = kb % p.stages, round = kb / p.stages;
        if (!mbar_wait(&full[st], round & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + st * kQkvABytes), b0 = smem_u32(xs + kb * kQkvBBytes);
#pragma unroll
        for (int k = 0; k < kQkvTileK / 16; ++k)
          umma_bf16(tmem_base, umma_sdesc_sw128(a0 + k * 32), umma_sdesc_sw128(b0 + k * 32), IDESC,
                    (kb > 0 || k > 0) ? 1u : 0u);
        umma_commit(&empty[st]);
      }
      umma_commit(accf);  // arrives once every MMA issued has completed (also after an abort)
    }
    __syncwarp();
  }
  // epilogue: thread t holds output column m0 + t (TMEM lane t), batch rows in columns 0 .. 15
  const bool ok = __all_sync(0xffffffffu, mbar_wait(accf, 0, abort_flag) && *abort_flag == 0);
  tc_fence_after();
  float v[kQkvN];
  if (ok) {
    tmem_ld16(tmem_base + ((uint32_t)(warp * 32) << 16), v);
  } else {
#pragma unroll
    for (int b = 0; b < kQkvN; ++b) v[b] = 0.f;
  }
  const int n = m0 + threadIdx.x;
  const int pos = qkv_position(p);
  float* part = reinterpret_cast<float*>(smem + qkv_mma_part_offset(p.stages, p.kbs_max)) + threadIdx.x;
#pragma unroll
  for (int b = 0; b < kQkvN; ++b) part[b * kQkvTileM] = v[b];
  cluster_sync_all();  // every split's partial tile is in place
  for (int b = split; b < p.batch; b += p.splits) {
    float pv[kQkvMaxSplits];
#pragma unroll
    for (int r = 0; r < kQkvMaxSplits; ++r) pv[r] = r < p.splits ? ld_dsmem_f32(part + b * kQkvTileM, r) : 0.f;
    float acc = pv[0];
#pragma unroll
    for (int r = 1; r < kQkvMaxSplits; ++r)
      if (r < p.splits) acc += pv[r];
    if (n < p.n_cols) qkv_store(p, n, b, pos, acc);
  }
  cluster_sync_all();  // no CTA leaves while a peer may still read its partial
  tc_fence_before();
  __syncthreads();
  if (*abort_flag != 0) {
    if (threadIdx.x == 0) {
      flag_status(p.status, SAGA_STATUS_TIMEOUT);
      for (int t = (issued > p.stages ? issued - p.stages : 0); t < issued; ++t)
        mbar_wait_drain(&full[t % p.stages], (t / p.stages) & 1);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ============================================================================ launchers
// Every kernel is launched with programmatic stream serialization: it may
// start while the previous kernel on the stream finishes, runs its
// independent setup, and waits (pdl_wait) before touching shared data.
// SAGA_PDL=0 in the environment turns this off (plain stream order).
static bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("SAGA_PDL");
    return !(e != nullptr && e[0] == '0');
  }();
  return on;
}

template <typename... KArgs, typename... Args>
static cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                            Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// cudaFuncSetAttribute holds per device: one bit per device ordinal.
// Per kernel and device, once: the dynamic shared memory it may take, and
// the largest shared-memory carveout.  Every kernel of the library asks for
// the same carveout, so an SM running a small kernel (a combine) never has
// to drain and reconfigure before a split CTA of the next call can join it.
static cudaError_t ensure_smem(const void* fn, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  if (bytes > 0) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
  return e;
}

template <int D, int NP, bool UMMA, bool DUMP>
static cudaError_t run_split(const CUtensorMap& tf, const CUtensorMap& tp, const SplitParams& p, dim3 grid,
                             cudaStream_t st, int* occ) {
  using K = SplitSmem<D, NP, UMMA>;
  static std::atomic<uint64_t> prepared{0};
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(saga_split_kernel<D, NP, UMMA, DUMP>), K::ALLOC, prepared);
  if (e != cudaSuccess) return e;
  if (occ != nullptr)
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, saga_split_kernel<D, NP, UMMA, DUMP>, 192, K::ALLOC);
  return launch_k(saga_split_kernel<D, NP, UMMA, DUMP>, grid, dim3(192), K::ALLOC, st, tf, tp, p);
}

template <int D>
static cudaError_t dispatch_np(int NP, bool dump, const CUtensorMap& tf, const CUtensorMap& tp, const SplitParams& p,
                               dim3 g, cudaStream_t st, int* occ) {
  switch (NP) {
    case 4: return dump ? run_split<D, 4, true, true>(tf, tp, p, g, st, occ) : run_split<D, 4, true, false>(tf, tp, p, g, st, occ);
    case 8: return dump ? run_split<D, 8, true, true>(tf, tp, p, g, st, occ) : run_split<D, 8, true, false>(tf, tp, p, g, st, occ);
    case 16: return dump ? run_split<D, 16, true, true>(tf, tp, p, g, st, occ) : run_split<D, 16, true, false>(tf, tp, p, g, st, occ);
    case 32: return dump ? run_split<D, 32, true, true>(tf, tp, p, g, st, occ) : run_split<D, 32, true, false>(tf, tp, p, g, st, occ);
    case 64:
      if constexpr (D == 64) {
        return dump ? run_split<D, 64, true, true>(tf, tp, p, g, st, occ) : run_split<D, 64, true, false>(tf, tp, p, g, st, occ);
      } else {
        return cudaErrorInvalidValue;  // d = 128 supports at most 32 query heads per key head
      }
    default:
      return cudaErrorInvalidValue;
  }
}

// mode: kSplitDense / kSplitSparse attend (they differ only in p.tau, null
// for dense), kSplitDump dumps scores for a refresh.
cudaError_t launch_split(int D, int NP, int mode, const CUtensorMap& tf, const CUtensorMap& tp, const SplitParams& p,
                         dim3 grid, cudaStream_t st, int* occupancy_out) {
  const bool dump = mode == kSplitDump;
  if (D == 64) return dispatch_np<64>(NP, dump, tf, tp, p, grid, st, occupancy_out);
  if (D == 128) return dispatch_np<128>(NP, dump, tf, tp, p, grid, st, occupancy_out);
  return cudaErrorInvalidValue;
}

template <int D, int NP>
static cudaError_t run_from_scores(const SplitParams& p, dim3 grid, cudaStream_t st, int* occ) {
  static std::atomic<uint64_t> prepared{0};
  const int bytes = FromScoresSmem<D, NP>::BYTES;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(saga_from_scores_kernel<D, NP>), bytes, prepared);
  if (e != cudaSuccess) return e;
  if (occ != nullptr)
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, saga_from_scores_kernel<D, NP>, kEpiThreads, bytes);
  return launch_k(saga_from_scores_kernel<D, NP>, grid, dim3(kEpiThreads), bytes, st, p);
}

template <int D, int NP>
static cudaError_t run_dense(const CUtensorMap& kf, const CUtensorMap& kp, const CUtensorMap& vf, const CUtensorMap& vp,
                             const SplitParams& p, dim3 grid, cudaStream_t st, int* occ) {
  using K = DenseSmem<D, NP>;
  static std::atomic<uint64_t> prepared{0};
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(saga_dense_kernel<D, NP>), K::ALLOC, prepared);
  if (e != cudaSuccess) return e;
  if (occ != nullptr)
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, saga_dense_kernel<D, NP>, K::THREADS, K::ALLOC);
  return launch_k(saga_dense_kernel<D, NP>, grid, dim3(K::THREADS), K::ALLOC, st, kf, kp, vf, vp, p);
}

// Dense attention (every token kept) for groups whose query heads share one
// value head; NP in {4, 8, 16}.
cudaError_t launch_dense(int D, int NP, const CUtensorMap& kf, const CUtensorMap& kp, const CUtensorMap& vf,
                         const CUtensorMap& vp, const SplitParams& p, dim3 grid, cudaStream_t st, int* occ) {
#define SAGA_DN(DD, NN) \
  if (D == DD && NP == NN) return run_dense<DD, NN>(kf, kp, vf, vp, p, grid, st, occ);
  SAGA_DN(64, 4) SAGA_DN(64, 8) SAGA_DN(64, 16) SAGA_DN(128, 4) SAGA_DN(128, 8) SAGA_DN(128, 16)
#undef SAGA_DN
  return cudaErrorInvalidValue;
}

cudaError_t launch_from_scores(int D, int NP, const SplitParams& p, dim3 grid, cudaStream_t st, int* occ) {
#define SAGA_FS(DD, NN) \
  if (D == DD && NP == NN) return run_from_scores<DD, NN>(p, grid, st, occ);
  SAGA_FS(64, 4) SAGA_FS(64, 8) SAGA_FS(64, 16) SAGA_FS(64, 32) SAGA_FS(64, 64)
  SAGA_FS(128, 4) SAGA_FS(128, 8) SAGA_FS(128, 16) SAGA_FS(128, 32)
#undef SAGA_FS
  return cudaErrorInvalidValue;
}

cudaError_t launch_combine(int D, const CombineParams& p, cudaStream_t st) {
  static std::atomic<uint64_t> prepared64{0}, prepared128{0};
  cudaError_t e;
  if (D == 64) {
    e = ensure_smem(reinterpret_cast<const void*>(saga_combine_kernel<64>), 0, prepared64);
    if (e != cudaSuccess) return e;
    return launch_k(saga_combine_kernel<64>, dim3(p.rows, 2), dim3(kCombineThreads), 0, st, p);
  }
  if (D == 128) {
    e = ensure_smem(reinterpret_cast<const void*>(saga_combine_kernel<128>), 0, prepared128);
    if (e != cudaSuccess) return e;
    return launch_k(saga_combine_kernel<128>, dim3(p.rows, 4), dim3(kCombineThreads), 0, st, p);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_select(const SelectParams& p, int rows, cudaStream_t st) {
  static std::atomic<uint64_t> prepared{0};
  const int bytes = kSelectCap * 4;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(atopn_select_kernel), bytes, prepared);
  if (e != cudaSuccess) return e;
  return launch_k(atopn_select_kernel, dim3(rows), dim3(kSelectThreads), bytes, st, p);
}

// The refresh path's select for a few long rows: one cluster of CTAs per row.
cudaError_t launch_select_cluster(const SelectParams& p, int rows, cudaStream_t st) {
  static std::atomic<uint64_t> prepared{0};
  const int bytes = kSelectCap * 4;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(atopn_cluster_select_kernel), bytes, prepared);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kSelCluster, rows);
  cfg.blockDim = dim3(kSelClusterThreads);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kSelCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, atopn_cluster_select_kernel, p);
}

template <int NB>
static cudaError_t run_qkv(const QkvParams& p, cudaStream_t st) {
  static std::atomic<uint64_t> prepared{0};
  const int bytes = NB * kQkvChunk * 2;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(saga_qkv_kernel<NB>), bytes, prepared);
  if (e != cudaSuccess) return e;
  return launch_k(saga_qkv_kernel<NB>, dim3((p.n_cols + kQkvWarps - 1) / kQkvWarps), dim3(kQkvWarps * 32), bytes, st,
                  p);
}

// The QKV projection: batch 1 on CUDA cores, batch 2 .. 16 on the tensor cores.
cudaError_t launch_qkv(const QkvParams& p, const CUtensorMap& tw, cudaStream_t st) {
  if (p.batch < kQkvMmaMinBatch) {
    if (p.batch <= 1) return run_qkv<1>(p, st);
    if (p.batch <= 2) return run_qkv<2>(p, st);
    if (p.batch <= 4) return run_qkv<4>(p, st);
    if (p.batch <= 8) return run_qkv<8>(p, st);
    return run_qkv<16>(p, st);
  }
  static std::atomic<uint64_t> prepared{0};
  const int bytes = qkv_mma_smem_bytes(p.stages, p.kbs_max);
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(saga_qkv_mma_kernel), qkv_mma_smem_bytes(kQkvMaxStages, kQkvMaxKb),
                              prepared);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.splits, (p.n_cols + kQkvTileM - 1) / kQkvTileM);
  cfg.blockDim = dim3(kQkvMmaThreads);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;  // the splits of a tile: one cluster
  attr[0].val.clusterDim.x = p.splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, saga_qkv_mma_kernel, tw, p);
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t st) {
  static std::atomic<uint64_t> prepared{0};
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(saga_append_kernel), 0, prepared);
  if (e != cudaSuccess) return e;
  const int n = p.batch * (p.h_k + p.h_v) * (p.d / 8);
  return launch_k(saga_append_kernel, dim3((n + 255) / 256), dim3(256), 0, st, p);
}

cudaError_t launch_fill(float* dst, float v, int n, cudaStream_t st) {
  static std::atomic<uint64_t> prepared{0};
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(saga_fill_kernel), 0, prepared);
  if (e != cudaSuccess) return e;
  return launch_k(saga_fill_kernel, dim3((n + 255) / 256), dim3(256), 0, st, dst, v, n);
}

}  // namespace saga
