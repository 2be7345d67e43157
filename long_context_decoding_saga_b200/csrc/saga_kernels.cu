// saga_kernels.cu - the SAGA + Atop-N decode-attention kernels for sm_100a.
//
// One decode step of one layer ("More Value per Key: Asymmetric Sparse
// Attention for Faster LLM Decoding"):
//   split kernel   : per (batch, key head, context split) CTA.  A TMA producer
//                    streams 128-token key tiles into a 128-byte-swizzled
//                    shared-memory ring; scores A = q K^T / sqrt(d) (eq. 2)
//                    for all query heads of the key head come from one
//                    tcgen05.mma per 16 dims (keys = M 128, queries = N) into
//                    TMEM, or from CUDA-core FMAs for groups of <= 4 query
//                    heads; four epilogue warps compare against the Atop-N
//                    threshold (Atop-N step 1), compact the kept tokens with
//                    ballots and prefix sums, and accumulate the sparse
//                    softmax and value sum of eq. 7 online over the h_v value
//                    heads, writing one (max, sum, o) partial per split.
//   dump variant   : refresh steps (Atop-N step 2) - the same scores are
//                    written out with a per-head histogram of their top byte.
//   select kernel  : exact N-th largest score per row by radix selection.
//   from-scores    : refresh steps - compare/gather from the dumped scores.
//   combine kernel : merges the split partials (log-sum-exp) into O.
//   append kernel  : writes the new token's key/value rows into the cache.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "saga_device.cuh"
#include "saga_internal.h"

namespace saga {

// ============================================================================ helpers
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

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

// Time-bounded wait that ignores the abort flag (used to drain in-flight copies).
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 63u && global_ns() - t0 > kWaitLimitNs) return false;
  }
}

template <int D>
__host__ __device__ constexpr int split_stages() { return D == 128 ? 4 : 6; }

template <int NP>
__host__ __device__ constexpr uint32_t tmem_cols() { return (2 * NP <= 32) ? 32u : (2 * NP <= 64) ? 64u : 128u; }

// ============================================================================ epilogue
// Per-tile staging: union rows (tokens kept by at least one query head of the
// group), their value-head bits and softmax weights, written in phase A of a
// tile and consumed by phase B one tile later (so the L2 prefetch of the
// value rows issued in phase A overlaps the next tile's key stream).
template <int NP>
struct EpiSlot {
  float w[kTile][NP];
  int tok[kTile];
  uint32_t vmask[kTile];
  float factor[NP];
  int nrows;
  int active;
};

constexpr int kRedFloats = 2048;  // G*D bound when row groups are reduced (see EpiCtx)

template <int NP>
struct EpiShared {
  EpiSlot<NP> slot[2];
  float tau[NP];
  float m_run[NP];
  float wmax[4][NP];
  int wrows[4];
  int hcnt[4][NP];
  int cnt_run[NP];
  float red_o[kRedFloats];
  float red_l[kMaxG];
};

constexpr int kPT = 4;  // phase-B ownership slots per thread

// Phase-B ownership: thread et accumulates, for pair (value head u, 4-dim
// chunk c, block hb of up to 4 query heads of u) and row group rg, the
// running numerator and denominator of eq. 7.
template <int D>
struct EpiCtx {
  int et, q, lane, erow;
  int G, nvh, hpv, hb_n, P, RG;
  int valid[kPT], u[kPT], c[kPT], hb[kPT], rg[kPT];

  __device__ void init(int et_, int G_, int nvh_, int hpv_) {
    et = et_;
    lane = et_ & 31;
    q = (threadIdx.x >> 5) & 3;
    erow = 32 * q + lane;
    G = G_;
    nvh = nvh_;
    hpv = hpv_;
    hb_n = (hpv + 3) / 4;
    P = nvh * (D / 4) * hb_n;
    RG = P < kEpiThreads ? kEpiThreads / P : 1;
    const int W = P * RG;
#pragma unroll
    for (int i = 0; i < kPT; ++i) {
      const int s = et + kEpiThreads * i;
      valid[i] = s < W;
      const int pair = s % P;
      rg[i] = s / P;
      c[i] = pair % (D / 4);
      const int rest = pair / (D / 4);
      hb[i] = rest % hb_n;
      u[i] = rest / hb_n;
    }
  }
};

struct EpiAcc {
  float o[kPT][4][4];
  float l[kPT][4];
  __device__ void zero() {
#pragma unroll
    for (int i = 0; i < kPT; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        l[i][k] = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) o[i][k][e] = 0.f;
      }
  }
};

template <int NP>
__device__ void epi_setup(EpiShared<NP>& es, int et, const SplitParams& p, int b, int j0, bool load_tau) {
  if (et < NP) {
    es.tau[et] = (load_tau && et < p.G) ? p.tau[(size_t)b * p.h_q + j0 + et] : INFINITY;
    es.m_run[et] = -INFINITY;
    es.cnt_run[et] = 0;
  }
  for (int i = et; i < kRedFloats; i += kEpiThreads) es.red_o[i] = 0.f;
  if (et < kMaxG) es.red_l[et] = 0.f;
}

// Phase A of tile `slot_i`: threshold compare (Atop-N step 1), per-head tile
// max, compaction of the union rows, softmax weights, L2 prefetch of the
// value rows, and (optionally) per-head counts and ascending index lists.
template <int D, int NP>
__device__ void phase_a(EpiShared<NP>& es, int slot_i, const float (&sc)[NP], int tok, bool valid, const EpiCtx<D>& cx,
                        const SplitParams& p, int b, int j0, int chunk_start, const uint16_t* vgroup) {
  EpiSlot<NP>& sl = es.slot[slot_i];
  uint64_t keep = 0;
#pragma unroll
  for (int jl = 0; jl < NP; ++jl)
    if (jl < cx.G && valid && sc[jl] >= es.tau[jl]) keep |= 1ull << jl;
  const bool any = named_bar_or(1, kEpiThreads, keep != 0);
  if (!any) {
    if (cx.et == 0) sl.active = 0;
    return;
  }
#pragma unroll
  for (int jl = 0; jl < NP; ++jl) {
    if (jl < cx.G) {
      float v = ((keep >> jl) & 1ull) ? sc[jl] : -INFINITY;
      v = warp_max(v);
      if (cx.lane == 0) es.wmax[cx.q][jl] = v;
    }
  }
  const bool isrow = keep != 0;
  const uint32_t bal = __ballot_sync(0xffffffffu, isrow);
  if (cx.lane == 0) es.wrows[cx.q] = __popc(bal);
  named_bar_sync(1, kEpiThreads);
  if (cx.et < cx.G) {
    const int jl = cx.et;
    const float tmax = fmaxf(fmaxf(es.wmax[0][jl], es.wmax[1][jl]), fmaxf(es.wmax[2][jl], es.wmax[3][jl]));
    const float mold = es.m_run[jl];
    const float mnew = fmaxf(mold, tmax);
    sl.factor[jl] = (mnew == -INFINITY) ? 1.f : __expf(mold - mnew);
    es.m_run[jl] = mnew;
  }
  int base = 0;
  for (int qq = 0; qq < cx.q; ++qq) base += es.wrows[qq];
  const int total = es.wrows[0] + es.wrows[1] + es.wrows[2] + es.wrows[3];
  named_bar_sync(1, kEpiThreads);
  if (isrow) {
    const int pos = base + __popc(bal & ((1u << cx.lane) - 1u));
    sl.tok[pos] = tok;
    uint32_t vm = 0;
#pragma unroll
    for (int jl = 0; jl < NP; ++jl) {
      if (jl < cx.G) {
        float w = 0.f;
        if ((keep >> jl) & 1ull) {
          w = __expf(sc[jl] - es.m_run[jl]);
          vm |= 1u << (jl / cx.hpv);
        }
        sl.w[pos][jl] = w;
      }
    }
    sl.vmask[pos] = vm;
    uint32_t bits = vm;
    while (bits) {
      const int u = __ffs(bits) - 1;
      bits &= bits - 1;
      prefetch_l2_bulk(vgroup + ((size_t)u * p.l_cap + tok) * D, D * 2);
    }
  }
  if (cx.et == 0) {
    sl.nrows = total;
    sl.active = 1;
  }
  if (p.want_counts) {
#pragma unroll
    for (int jl = 0; jl < NP; ++jl) {
      if (jl < cx.G) {
        const uint32_t bl = __ballot_sync(0xffffffffu, (keep >> jl) & 1ull);
        if (cx.lane == 0) es.hcnt[cx.q][jl] = __popc(bl);
      }
    }
    named_bar_sync(1, kEpiThreads);
    if (p.idxbuf != nullptr) {
#pragma unroll
      for (int jl = 0; jl < NP; ++jl) {
        if (jl < cx.G) {
          const bool kb = (keep >> jl) & 1ull;
          const uint32_t bl = __ballot_sync(0xffffffffu, kb);
          if (kb) {
            int off = es.cnt_run[jl];
            for (int qq = 0; qq < cx.q; ++qq) off += es.hcnt[qq][jl];
            off += __popc(bl & ((1u << cx.lane) - 1u));
            p.idxbuf[((size_t)b * p.h_q + j0 + jl) * p.l_cap + chunk_start + off] = tok;
          }
        }
      }
    }
    named_bar_sync(1, kEpiThreads);
    if (cx.et < cx.G)
      es.cnt_run[cx.et] += es.hcnt[0][cx.et] + es.hcnt[1][cx.et] + es.hcnt[2][cx.et] + es.hcnt[3][cx.et];
  }
}

// Phase B of tile `slot_i`: rescale the running sums to the new maxima and
// add w * V[row] for every kept (row, query head) this thread owns.
template <int D, int NP>
__device__ void phase_b(EpiShared<NP>& es, int slot_i, const EpiCtx<D>& cx, const uint16_t* vgroup, int l_cap,
                        EpiAcc& acc) {
  EpiSlot<NP>& sl = es.slot[slot_i];
  if (!sl.active) return;
  const int nrows = sl.nrows;
#pragma unroll
  for (int i = 0; i < kPT; ++i) {
    if (!cx.valid[i]) continue;
    const int u = cx.u[i];
    const int jb = u * cx.hpv + cx.hb[i] * 4;
    const int nk = min(4, cx.hpv - cx.hb[i] * 4);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k < nk) {
        const float f = sl.factor[jb + k];
        acc.l[i][k] *= f;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc.o[i][k][e] *= f;
      }
    }
    const uint16_t* vb = vgroup + (size_t)u * l_cap * D + cx.c[i] * 4;
    const int step = cx.RG;
    for (int r0 = cx.rg[i]; r0 < nrows; r0 += 4 * step) {
      uint2 raw[4];
      bool use[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int r = r0 + t * step;
        use[t] = (r < nrows) && ((sl.vmask[r] >> u) & 1u);
        if (use[t]) raw[t] = __ldg(reinterpret_cast<const uint2*>(vb + (size_t)sl.tok[r] * D));
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (!use[t]) continue;
        const int r = r0 + t * step;
        const float v0 = bf16_lo(raw[t].x), v1 = bf16_hi(raw[t].x), v2 = bf16_lo(raw[t].y), v3 = bf16_hi(raw[t].y);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (k < nk) {
            const float w = sl.w[r][jb + k];
            acc.l[i][k] += w;
            acc.o[i][k][0] = fmaf(w, v0, acc.o[i][k][0]);
            acc.o[i][k][1] = fmaf(w, v1, acc.o[i][k][1]);
            acc.o[i][k][2] = fmaf(w, v2, acc.o[i][k][2]);
            acc.o[i][k][3] = fmaf(w, v3, acc.o[i][k][3]);
          }
        }
      }
    }
  }
}

// Writes this split's partial (running max m, denominator l, numerator o)
// for every query head of the group.
template <int D, int NP>
__device__ void epi_finish(EpiShared<NP>& es, const EpiCtx<D>& cx, EpiAcc& acc, const SplitParams& p, int b, int j0,
                           int s) {
  const size_t row0 = (size_t)b * p.h_q + j0;
  if (cx.RG > 1) {
#pragma unroll
    for (int i = 0; i < kPT; ++i) {
      if (!cx.valid[i]) continue;
      const int jb = cx.u[i] * cx.hpv + cx.hb[i] * 4;
      const int nk = min(4, cx.hpv - cx.hb[i] * 4);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (k < nk) {
#pragma unroll
          for (int e = 0; e < 4; ++e) atomicAdd(&es.red_o[(jb + k) * D + cx.c[i] * 4 + e], acc.o[i][k][e]);
          if (cx.c[i] == 0) atomicAdd(&es.red_l[jb + k], acc.l[i][k]);
        }
      }
    }
    named_bar_sync(1, kEpiThreads);
    for (int idx = cx.et; idx < cx.G * (D / 4); idx += kEpiThreads) {
      const int jl = idx / (D / 4), c4 = idx % (D / 4);
      const float4 v = *reinterpret_cast<const float4*>(&es.red_o[jl * D + c4 * 4]);
      *reinterpret_cast<float4*>(&p.part_o[((row0 + jl) * p.s_cap + s) * D + c4 * 4]) = v;
    }
    if (cx.et < cx.G) p.part_l[(row0 + cx.et) * p.s_cap + s] = es.red_l[cx.et];
  } else {
#pragma unroll
    for (int i = 0; i < kPT; ++i) {
      if (!cx.valid[i]) continue;
      const int jb = cx.u[i] * cx.hpv + cx.hb[i] * 4;
      const int nk = min(4, cx.hpv - cx.hb[i] * 4);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (k < nk) {
          const size_t r = (row0 + jb + k) * p.s_cap + s;
          *reinterpret_cast<float4*>(&p.part_o[r * D + cx.c[i] * 4]) =
              make_float4(acc.o[i][k][0], acc.o[i][k][1], acc.o[i][k][2], acc.o[i][k][3]);
          if (cx.c[i] == 0) p.part_l[r] = acc.l[i][k];
        }
      }
    }
  }
  if (cx.et < cx.G) {
    p.part_m[(row0 + cx.et) * p.s_cap + s] = es.m_run[cx.et];
    p.part_cnt[(row0 + cx.et) * p.s_cap + s] = es.cnt_run[cx.et];
  }
}

// ============================================================================ split kernel
template <int D, int NP, bool UMMA>
struct SplitSmem {
  static constexpr int NATOM = D / 64;
  static constexpr int STAGE_BYTES = kTile * D * 2;
  static constexpr int NSTAGE = split_stages<D>();
  static constexpr int QBYTES = UMMA ? NATOM * NP * 128 : NP * D * 4;
  static constexpr int Q_OFF = NSTAGE * STAGE_BYTES;
  static constexpr int EPI_OFF = Q_OFF + ((QBYTES + 1023) / 1024) * 1024;
  static constexpr int BAR_OFF = EPI_OFF + ((int)sizeof(EpiShared<NP>) + 15) / 16 * 16;
  static constexpr int NBARS = 2 * NSTAGE + 5;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
};

template <int D, int NP, bool UMMA, bool DUMP>
__global__ void __launch_bounds__(192, 1)
    saga_split_kernel(const __grid_constant__ CUtensorMap tmap_full, const __grid_constant__ CUtensorMap tmap_part,
                      const SplitParams p) {
  using SM = SplitSmem<D, NP, UMMA>;
  constexpr int NATOM = SM::NATOM;
  constexpr int NSTAGE = SM::NSTAGE;
  constexpr int STAGE_BYTES = SM::STAGE_BYTES;
  constexpr uint32_t TMEM_COLS = tmem_cols<NP>();
  constexpr uint32_t IDESC = umma_idesc_bf16(128, NP < 16 ? 16 : NP);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kst = smem;
  uint8_t* qsm = smem + SM::Q_OFF;
  EpiShared<NP>& es = *reinterpret_cast<EpiShared<NP>*>(smem + SM::EPI_OFF);
  uint32_t* hist = reinterpret_cast<uint32_t*>(&es.slot[0]);  // dump mode: [NP][256]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::BAR_OFF);
  uint64_t* empty = full + NSTAGE;
  uint64_t* accf = empty + NSTAGE;
  uint64_t* acce = accf + 2;
  uint64_t* fin = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::MISC_OFF + 4);

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = h * p.G;
  const int L = device_seq_len(p.seq_len_dev, p.seq_len, p.l_cap, (s == 0 && h == 0 && b == 0) ? p.status : nullptr);
  int start, end;
  split_range(L, p.nsplit, s, &start, &end);
  const int ntiles = (end - start + kTile - 1) / kTile;
  const int row_base = (b * p.h_k + h) * p.l_cap;  // first cache row of this (batch, key head)

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], UMMA ? 1 : 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accf[i], 1);
      mbar_init(&acce[i], 4);
    }
    mbar_init(fin, 1);
    mbar_init_fence();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_full);
    tma_prefetch_desc(&tmap_part);
  }
  if (UMMA && warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp >= 2) {
    const int et = threadIdx.x - 64;
    epi_setup<NP>(es, et, p, b, j0, !DUMP);
    if (UMMA) {
      // q as the K-major B operand in the 128-byte swizzle layout; rows >= G are zero
      for (int i = et; i < NATOM * NP * 8; i += kEpiThreads) {
        const int a = i / (NP * 8), n = (i / 8) % NP, c = i % 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < p.G) v = *reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.h_q + j0 + n) * D + a * 64 + c * 8);
        *reinterpret_cast<uint4*>(qsm + a * NP * 128 + n * 128 + ((c ^ (n & 7)) << 4)) = v;
      }
    } else {
      float* qf = reinterpret_cast<float*>(qsm);
      for (int i = et; i < NP * D; i += kEpiThreads) {
        const int n = i / D, k = i % D;
        float v = 0.f;
        if (n < p.G) v = __uint_as_float((uint32_t)p.q[((size_t)b * p.h_q + j0 + n) * D + k] << 16);
        qf[i] = v;
      }
    }
    if (DUMP)
      for (int i = et; i < NP * 256; i += kEpiThreads) hist[i] = 0u;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = UMMA ? *tmem_slot : 0u;

  int issued = 0;  // producer: tiles issued
  // ---------------------------------------------------------------- roles
  if (warp == 0) {
    if (lane == 0) {
      for (int t = 0; t < ntiles; ++t) {
        const int stage = t % NSTAGE, round = t / NSTAGE;
        if (round > 0 && !mbar_wait(&empty[stage], (round - 1) & 1, abort_flag)) break;
        const int r0 = start + t * kTile;
        const int rows = min(kTile, end - r0);
        uint8_t* dst = kst + stage * STAGE_BYTES;
        if (rows == kTile) {
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
#pragma unroll
          for (int a = 0; a < NATOM; ++a) tma_load_2d(dst + a * 16384, &tmap_full, &full[stage], a * 64, row_base + r0);
        } else {
          const int nsub = (rows + kUnit - 1) / kUnit;
          mbar_arrive_expect_tx(&full[stage], nsub * kUnit * 128 * NATOM);
          for (int i = 0; i < nsub; ++i)
#pragma unroll
            for (int a = 0; a < NATOM; ++a)
              tma_load_2d(dst + a * 16384 + i * kUnit * 128, &tmap_part, &full[stage], a * 64,
                          row_base + r0 + i * kUnit);
        }
        issued = t + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (UMMA && lane == 0) {
      for (int t = 0; t < ntiles; ++t) {
        const int stage = t % NSTAGE, round = t / NSTAGE;
        if (!mbar_wait(&full[stage], round & 1, abort_flag)) break;
        const int abuf = t & 1;
        if (t >= 2 && !mbar_wait(&acce[abuf], ((t >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(kst + stage * STAGE_BYTES);
        const uint32_t b0 = smem_u32(qsm);
        const uint32_t d_tmem = tmem_base + abuf * NP;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t aa = a0 + (k >> 2) * 16384 + (k & 3) * 32;
          const uint32_t bb = b0 + (k >> 2) * NP * 128 + (k & 3) * 32;
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
    EpiCtx<D> cx;
    const int v_base = (int)(((long long)j0 * p.h_v) / p.h_q);
    cx.init(et, p.G, p.nvh, p.hpv);
    EpiAcc acc;
    acc.zero();
    const uint16_t* vgroup = p.v_cache + ((size_t)b * p.h_v + v_base) * (size_t)p.l_cap * D;
    const size_t srow = ((size_t)b * p.h_q + j0) * (size_t)p.ld_scores;
    bool ok = true;
    int t = 0;
    for (; t < ntiles; ++t) {
      float sc[NP];
      if (UMMA) {
        const int abuf = t & 1;
        ok = mbar_wait(&accf[abuf], (t >> 1) & 1, abort_flag);
        ok = named_bar_and(1, kEpiThreads, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(32 * cx.q) << 16) + (uint32_t)(abuf * NP);
#pragma unroll
        for (int i = 0; i < NP / 16; ++i) tmem_ld16(taddr + 16 * i, sc + 16 * i);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[abuf]);
      } else {
        const int stage = t % NSTAGE;
        ok = mbar_wait(&full[stage], (t / NSTAGE) & 1, abort_flag);
        ok = named_bar_and(1, kEpiThreads, ok);
        if (!ok) break;
        const uint8_t* rowp = kst + stage * STAGE_BYTES + cx.erow * 128;
        const float* qf = reinterpret_cast<const float*>(qsm);
#pragma unroll
        for (int n = 0; n < NP; ++n) sc[n] = 0.f;
#pragma unroll
        for (int a = 0; a < NATOM; ++a) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 raw = *reinterpret_cast<const uint4*>(rowp + a * 16384 + ((c ^ (cx.erow & 7)) << 4));
            const float kv[8] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y),
                                 bf16_lo(raw.z), bf16_hi(raw.z), bf16_lo(raw.w), bf16_hi(raw.w)};
#pragma unroll
            for (int n = 0; n < NP; ++n) {
              const float4 qa = *reinterpret_cast<const float4*>(qf + n * D + a * 64 + c * 8);
              const float4 qb = *reinterpret_cast<const float4*>(qf + n * D + a * 64 + c * 8 + 4);
              float x = sc[n];
              x = fmaf(kv[0], qa.x, x);
              x = fmaf(kv[1], qa.y, x);
              x = fmaf(kv[2], qa.z, x);
              x = fmaf(kv[3], qa.w, x);
              x = fmaf(kv[4], qb.x, x);
              x = fmaf(kv[5], qb.y, x);
              x = fmaf(kv[6], qb.z, x);
              x = fmaf(kv[7], qb.w, x);
              sc[n] = x;
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
      }
#pragma unroll
      for (int n = 0; n < NP; ++n) sc[n] *= p.scale;
      const int tok = start + t * kTile + cx.erow;
      const bool valid = tok < end;
      if (DUMP) {
#pragma unroll
        for (int jl = 0; jl < NP; ++jl) {
          if (jl < p.G) {
            if (valid) p.scores_out[srow + (size_t)jl * p.ld_scores + tok] = sc[jl];
            const uint32_t bin = valid ? (float_key(sc[jl]) >> 24) : 256u;
            const uint32_t peers = __match_any_sync(0xffffffffu, bin);
            if (valid && lane == __ffs(peers) - 1) atomicAdd(&hist[jl * 256 + bin], (uint32_t)__popc(peers));
          }
        }
      } else {
        phase_a<D, NP>(es, t & 1, sc, tok, valid, cx, p, b, j0, start, vgroup);
        if (t > 0) phase_b<D, NP>(es, (t - 1) & 1, cx, vgroup, p.l_cap, acc);
      }
    }
    if (!DUMP) {
      if (ok && ntiles > 0) {
        named_bar_sync(1, kEpiThreads);
        phase_b<D, NP>(es, (ntiles - 1) & 1, cx, vgroup, p.l_cap, acc);
      }
      named_bar_sync(1, kEpiThreads);
      epi_finish<D, NP>(es, cx, acc, p, b, j0, s);
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
  if (DUMP && warp >= 2) {
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
// compare and gather from them (same epilogue as the split kernel).
template <int D, int NP>
__global__ void __launch_bounds__(kEpiThreads) saga_from_scores_kernel(const SplitParams p) {
  extern __shared__ uint8_t smem_raw[];
  EpiShared<NP>& es = *reinterpret_cast<EpiShared<NP>*>(smem_raw);
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int et = threadIdx.x;
  const int j0 = h * p.G;
  const int L = device_seq_len(p.seq_len_dev, p.seq_len, p.l_cap, nullptr);
  int start, end;
  split_range(L, p.nsplit, s, &start, &end);
  const int ntiles = (end - start + kTile - 1) / kTile;

  epi_setup<NP>(es, et, p, b, j0, true);
  EpiCtx<D> cx;
  cx.init(et, p.G, p.nvh, p.hpv);
  EpiAcc acc;
  acc.zero();
  const int v_base = (int)(((long long)j0 * p.h_v) / p.h_q);
  const uint16_t* vgroup = p.v_cache + ((size_t)b * p.h_v + v_base) * (size_t)p.l_cap * D;
  const float* srow = p.scores_in + ((size_t)b * p.h_q + j0) * (size_t)p.ld_scores;
  __syncthreads();

  float nxt[NP];
  auto load = [&](int t, float (&dst)[NP]) {
    const int tok = start + t * kTile + cx.erow;
#pragma unroll
    for (int jl = 0; jl < NP; ++jl)
      dst[jl] = (jl < p.G && tok < end) ? __ldg(srow + (size_t)jl * p.ld_scores + tok) : -INFINITY;
  };
  if (ntiles > 0) load(0, nxt);
  for (int t = 0; t < ntiles; ++t) {
    float sc[NP];
#pragma unroll
    for (int jl = 0; jl < NP; ++jl) sc[jl] = nxt[jl];
    if (t + 1 < ntiles) load(t + 1, nxt);
    const int tok = start + t * kTile + cx.erow;
    named_bar_sync(1, kEpiThreads);
    phase_a<D, NP>(es, t & 1, sc, tok, tok < end, cx, p, b, j0, start, vgroup);
    if (t > 0) phase_b<D, NP>(es, (t - 1) & 1, cx, vgroup, p.l_cap, acc);
  }
  if (ntiles > 0) {
    named_bar_sync(1, kEpiThreads);
    phase_b<D, NP>(es, (ntiles - 1) & 1, cx, vgroup, p.l_cap, acc);
  }
  named_bar_sync(1, kEpiThreads);
  epi_finish<D, NP>(es, cx, acc, p, b, j0, s);
}

// ============================================================================ combine kernel
// O[b, j] = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s over the splits of
// row (b, j); zero when nothing was kept.  Also the kept counts and the
// ascending index list (concatenation of the per-split lists in split order).
constexpr int kCombineThreads = 512;

template <int D>
__global__ void __launch_bounds__(kCombineThreads) saga_combine_kernel(const CombineParams p) {
  constexpr int DPL = D / 32;  // dims per lane
  constexpr int NW = kCombineThreads / 32;
  __shared__ float red_m[NW];
  __shared__ float wsum[NW];
  __shared__ float wacc[NW][D];
  __shared__ int cnt_scan[kCombineThreads];
  const int row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.nsplit;
  const float* pm = p.part_m + (size_t)row * p.s_cap;
  const float* pl = p.part_l + (size_t)row * p.s_cap;
  const float* po = p.part_o + (size_t)row * p.s_cap * D;

  float m = -INFINITY;
  for (int s = threadIdx.x; s < S; s += kCombineThreads) m = fmaxf(m, pm[s]);
  m = warp_max(m);
  if (lane == 0) red_m[warp] = m;
  __syncthreads();
  float M = red_m[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) M = fmaxf(M, red_m[w]);

  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  float den = 0.f;
  if (M != -INFINITY) {
    for (int s = warp; s < S; s += NW) {
      const float ms = pm[s];
      if (ms == -INFINITY) continue;
      const float f = __expf(ms - M);
      den = fmaf(f, pl[s], den);
      const float* src = po + (size_t)s * D + lane * DPL;
      if (DPL == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] = fmaf(f, v.x, acc[0]);
        acc[1] = fmaf(f, v.y, acc[1]);
        acc[2] = fmaf(f, v.z, acc[2]);
        acc[3] = fmaf(f, v.w, acc[3]);
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        acc[0] = fmaf(f, v.x, acc[0]);
        acc[1] = fmaf(f, v.y, acc[1]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < DPL; ++e) wacc[warp][lane * DPL + e] = acc[e];
  if (lane == 0) wsum[warp] = den;
  __syncthreads();
  if (threadIdx.x < D) {
    float num = 0.f, dd = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      num += wacc[w][threadIdx.x];
      dd += wsum[w];
    }
    const float o = (M == -INFINITY || dd <= 0.f) ? 0.f : num / dd;
    if (p.out_bf16) {
      reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)row * D + threadIdx.x] = __float2bfloat16_rn(o);
    } else {
      reinterpret_cast<float*>(p.out)[(size_t)row * D + threadIdx.x] = o;
    }
  }
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
        split_range(L, S, ss, &st, &en);
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
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool valid) {
  const uint32_t key = valid ? bin : 0xFFFFFFFFu;
  const uint32_t peers = __match_any_sync(0xffffffffu, key);
  if (valid && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

// Calls f(key, valid) for every element of row[0, L) with warp-uniform trip
// counts (so f may use full-warp primitives).  row is 16-byte aligned.
template <typename F>
__device__ __forceinline__ void scan_row(const float* row, int L, F&& f) {
  const int nvec = L >> 2;
  const int nvec_pad = (nvec + 31) & ~31;
  const float4* row4 = reinterpret_cast<const float4*>(row);
  for (int i = threadIdx.x; i < nvec_pad; i += kSelectThreads) {
    const bool inb = i < nvec;
    const float4 v = inb ? __ldg(row4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    f(float_key(v.x), inb);
    f(float_key(v.y), inb);
    f(float_key(v.z), inb);
    f(float_key(v.w), inb);
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
  int L = p.row_len;
  if (p.seq_len_dev != nullptr) L = device_seq_len(p.seq_len_dev, p.row_len, p.l_cap, nullptr);
  if (p.n_top >= L) {
    if (threadIdx.x == 0) p.tau[r] = -INFINITY;
    return;
  }
  const float* row = p.scores + (size_t)r * p.ld;

  for (int i = threadIdx.x; i < 256; i += kSelectThreads)
    hist[i] = p.hist != nullptr ? p.hist[(size_t)r * 256 + i] : 0u;
  if (threadIdx.x == 0) {
    ncand = 0;
    s_bin = 0;
    s_rank = 1;
    s_cnt = 0;
  }
  __syncthreads();
  if (p.hist == nullptr) {  // top digit histogram
    scan_row(row, L, [&](uint32_t k, bool ok) { hist_add(hist, k >> 24, ok); });
    __syncthreads();
  }
  find_bin(hist, (uint32_t)p.n_top, &s_bin, &s_rank, &s_cnt);
  __syncthreads();
  uint32_t prefix = s_bin << 24, mask = 0xFF000000u, rank = s_rank, cnt = s_cnt;
  bool in_smem = false;
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

// ============================================================================ append + fill
__global__ void saga_append_kernel(const AppendParams p) {
  const int chunks_row = p.d / 8;  // 16-byte chunks per row
  const int nk = p.batch * p.h_k * chunks_row, nv = p.batch * p.h_v * chunks_row;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
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
  if (i < n) dst[i] = v;
}

// ============================================================================ launchers
template <int D, int NP, bool UMMA, bool DUMP>
static cudaError_t prep_split() {
  static bool done = false;
  if (done) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(saga_split_kernel<D, NP, UMMA, DUMP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SplitSmem<D, NP, UMMA>::ALLOC);
  if (e == cudaSuccess) done = true;
  return e;
}

template <int D, int NP, bool UMMA, bool DUMP>
static cudaError_t run_split(const CUtensorMap& tf, const CUtensorMap& tp, const SplitParams& p, dim3 grid,
                             cudaStream_t st, int* occ) {
  cudaError_t e = prep_split<D, NP, UMMA, DUMP>();
  if (e != cudaSuccess) return e;
  if (occ != nullptr)
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, saga_split_kernel<D, NP, UMMA, DUMP>, 192,
                                                         SplitSmem<D, NP, UMMA>::ALLOC);
  saga_split_kernel<D, NP, UMMA, DUMP><<<grid, 192, SplitSmem<D, NP, UMMA>::ALLOC, st>>>(tf, tp, p);
  return cudaGetLastError();
}

template <int D, bool DUMP>
static cudaError_t dispatch_np(int NP, const CUtensorMap& tf, const CUtensorMap& tp, const SplitParams& p, dim3 g,
                               cudaStream_t st, int* occ) {
  switch (NP) {
    case 4: return run_split<D, 4, false, DUMP>(tf, tp, p, g, st, occ);
    case 16: return run_split<D, 16, true, DUMP>(tf, tp, p, g, st, occ);
    case 32: return run_split<D, 32, true, DUMP>(tf, tp, p, g, st, occ);
    case 64: return run_split<D, 64, true, DUMP>(tf, tp, p, g, st, occ);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_split(int D, int NP, bool dump, const CUtensorMap& tf, const CUtensorMap& tp, const SplitParams& p,
                         dim3 grid, cudaStream_t st, int* occupancy_out) {
  if (D == 64) return dump ? dispatch_np<64, true>(NP, tf, tp, p, grid, st, occupancy_out)
                           : dispatch_np<64, false>(NP, tf, tp, p, grid, st, occupancy_out);
  if (D == 128) return dump ? dispatch_np<128, true>(NP, tf, tp, p, grid, st, occupancy_out)
                            : dispatch_np<128, false>(NP, tf, tp, p, grid, st, occupancy_out);
  return cudaErrorInvalidValue;
}

template <int D, int NP>
static cudaError_t run_from_scores(const SplitParams& p, dim3 grid, cudaStream_t st) {
  static bool done = false;
  const int bytes = (int)sizeof(EpiShared<NP>);
  if (!done) {
    cudaError_t e = cudaFuncSetAttribute(saga_from_scores_kernel<D, NP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         bytes);
    if (e != cudaSuccess) return e;
    done = true;
  }
  saga_from_scores_kernel<D, NP><<<grid, kEpiThreads, bytes, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_from_scores(int D, int NP, const SplitParams& p, dim3 grid, cudaStream_t st) {
#define SAGA_FS(DD, NN) \
  if (D == DD && NP == NN) return run_from_scores<DD, NN>(p, grid, st);
  SAGA_FS(64, 4) SAGA_FS(64, 16) SAGA_FS(64, 32) SAGA_FS(64, 64)
  SAGA_FS(128, 4) SAGA_FS(128, 16) SAGA_FS(128, 32) SAGA_FS(128, 64)
#undef SAGA_FS
  return cudaErrorInvalidValue;
}

cudaError_t launch_combine(int D, const CombineParams& p, cudaStream_t st) {
  if (D == 64) saga_combine_kernel<64><<<p.rows, kCombineThreads, 0, st>>>(p);
  else if (D == 128) saga_combine_kernel<128><<<p.rows, kCombineThreads, 0, st>>>(p);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_select(const SelectParams& p, int rows, cudaStream_t st) {
  static bool done = false;
  const int bytes = kSelectCap * 4;
  if (!done) {
    cudaError_t e = cudaFuncSetAttribute(atopn_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    done = true;
  }
  atopn_select_kernel<<<rows, kSelectThreads, bytes, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t st) {
  const int n = p.batch * (p.h_k + p.h_v) * (p.d / 8);
  saga_append_kernel<<<(n + 255) / 256, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_fill(float* dst, float v, int n, cudaStream_t st) {
  saga_fill_kernel<<<(n + 255) / 256, 256, 0, st>>>(dst, v, n);
  return cudaGetLastError();
}

int epi_shared_bytes(int NP) {
  switch (NP) {
    case 4: return (int)sizeof(EpiShared<4>);
    case 16: return (int)sizeof(EpiShared<16>);
    case 32: return (int)sizeof(EpiShared<32>);
    case 64: return (int)sizeof(EpiShared<64>);
  }
  return 0;
}

}  // namespace saga
