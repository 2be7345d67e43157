// saga_merge.cu - the closed-form GQA-to-SAGA key-head merge on sm_100a.
//
// "More Value per Key: Asymmetric Sparse Attention for Faster LLM Decoding",
// Methodology > GQA-to-SAGA Conversion > Stage 1: a GQA model's h_k key heads
// are merged in pairs into h_k / 2 SAGA key heads.  For a pair (a, b) the
// merged key projection that minimises the squared logit error of eq. 13 is
// (Lemma 4.1, eq. 15)
//     M(a, b) = (W_K^a S_a + W_K^b S_b) (S_a + S_b)^+,   S_r = sum_{j of r} Q^j^T Q^j,
// and the pairing is the minimum-weight perfect matching of the complete
// graph with weights w(a, b) = L_ab(M(a, b)) (Theorem 4.2).
//
// Steps, each a kernel:
//   1. zero-padded transposes of X [T, D] and of every key head's queries
//      (the token axis becomes the contiguous one, so both operands of the
//      Gram products are K-major for tcgen05);
//   2. the Gram matrices G = X^T X [D, D] and S_r [d, d] on tcgen05 (bf16
//      products, fp32 accumulation in TMEM), one kernel for both;
//   3. per pair, in fp64: S = S_a + S_b, its eigen-decomposition by parallel
//      cyclic Jacobi rotations, the pseudoinverse, and the factors A, B of
//      M(a, b) = W_K^a A + W_K^b B;
//   4. G W_K^r per head, then per pair M(a, b) and the loss terms
//      tr(D^T G D S_r) with D = M(a, b) - W_K^r, r in {a, b} (eq. 13 through
//      the Gram matrices), in fp64;
//   5. the minimum-weight perfect matching by enumerating every matching,
//      and the merged projections of the chosen pairs.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "saga.h"
#include "saga_device.cuh"

namespace saga {
namespace merge {

constexpr int kTileMN = 128;  // GEMM output tile (UMMA M = N = 128)
constexpr int kTileK = 64;    // one 128-byte swizzle atom of bf16
constexpr int kStages = 4;
constexpr int kMaxHeads = 16;  // teacher key heads (the matching enumerates (h_k - 1)!! pairings)

__host__ __device__ inline long long round_up(long long x, long long m) { return (x + m - 1) / m * m; }

// ---------------------------------------------------------------- 1. transposes
// dst[z-th block][c][t] = src[t][c] for t < rows, c < cols: src row stride
// src_ld, z-th source block at src + z * src_zstride; the z-th destination
// block starts at (z / g) * group_stride + (z % g) * member_stride (so the g
// query heads of a key head lie side by side along the token axis).  The
// destination's padding is zeroed beforehand.
__global__ void merge_transpose_kernel(const uint16_t* __restrict__ src, int rows, int cols, long long src_ld,
                                       long long src_zstride, uint16_t* __restrict__ dst, long long dst_ld, int g,
                                       long long group_stride, long long member_stride) {
  __shared__ uint16_t tile[32][33];
  const int z = blockIdx.z;
  const uint16_t* s = src + (size_t)z * src_zstride;
  uint16_t* o = dst + (size_t)(z / g) * group_stride + (size_t)(z % g) * member_stride;
  const int c0 = blockIdx.x * 32, t0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int t = t0 + i, c = c0 + threadIdx.x;
    tile[i][threadIdx.x] = (t < rows && c < cols) ? s[(size_t)t * src_ld + c] : (uint16_t)0;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, t = t0 + threadIdx.x;
    if (c < cols && t < rows) o[(size_t)c * dst_ld + t] = tile[threadIdx.x][i];
  }
}

// ---------------------------------------------------------------- 2. Gram products on tcgen05
// C[z][m][n] = sum_k A[z*Mz + m][k] * B[z*Nz + n][k]: A and B bf16, K-major
// (behind 2-D tensor maps with 128-byte swizzle, boxes of 64 x 128), C fp32
// row-major with row stride ldc and block stride c_zstride.  One CTA per
// 128 x 128 tile: warp 0 issues the TMA loads into a 4-stage ring, warp 1
// the MMAs (M = N = 128, K = 16) into one TMEM accumulator, warps 2-5 read
// it back (one TMEM lane quarter each) and store fp32 rows.
struct GemmParams {
  int Mz, Nz;          // rows of A / B per batch entry (multiples of 128)
  int k_blocks;        // K / 64
  long long ldc, c_zstride;
  float* C;
  unsigned* status;
};

struct GemmSmem {
  static constexpr int TILE_BYTES = kTileMN * kTileK * 2;  // 16 KB
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int BAR_OFF = kStages * STAGE_BYTES;
  static constexpr int NBARS = 2 * kStages + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int ALLOC = BYTES + 1024;
};

__global__ void __launch_bounds__(192, 1)
    merge_gemm_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb, const GemmParams p) {
  using SM = GemmSmem;
  constexpr uint32_t IDESC = umma_idesc_bf16(kTileMN, kTileMN);
  constexpr uint32_t TMEM_COLS = kTileMN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::BAR_OFF);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint64_t* fin = accf + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::MISC_OFF + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * kTileMN, n0 = blockIdx.x * kTileMN, z = blockIdx.z;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(accf, 1);
    mbar_init(fin, 1);
    mbar_init_fence();
    tma_prefetch_desc(&ta);
    tma_prefetch_desc(&tb);
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

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = 0; kb < p.k_blocks; ++kb) {
        const int stage = kb % kStages, round = kb / kStages;
        if (round > 0 && !mbar_wait(&empty[stage], (round - 1) & 1, abort_flag)) break;
        uint8_t* dst = smem + stage * SM::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[stage], SM::STAGE_BYTES);
        tma_load_2d(dst, &ta, &full[stage], kb * kTileK, z * p.Mz + m0);
        tma_load_2d(dst + SM::TILE_BYTES, &tb, &full[stage], kb * kTileK, z * p.Nz + n0);
        issued = kb + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int kb = 0;
      for (; kb < p.k_blocks; ++kb) {
        const int stage = kb % kStages, round = kb / kStages;
        if (!mbar_wait(&full[stage], round & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + stage * SM::STAGE_BYTES);
        const uint32_t b0 = a0 + SM::TILE_BYTES;
#pragma unroll
        for (int k = 0; k < kTileK / 16; ++k)
          umma_bf16(tmem_base, umma_sdesc_sw128(a0 + k * 32), umma_sdesc_sw128(b0 + k * 32), IDESC,
                    (kb > 0 || k > 0) ? 1u : 0u);
        umma_commit(&empty[stage]);
      }
      umma_commit(accf);  // every MMA issued so far has completed (also on the abort path)
      umma_commit(fin);
      if (!mbar_wait_drain(fin, 0)) *abort_flag = 1;
    }
    __syncwarp();
  } else {
    const int q = warp & 3;  // TMEM lane quarter: rows 32q .. 32q+31 of the tile
    const bool ok = __all_sync(0xffffffffu, mbar_wait(accf, 0, abort_flag));
    if (ok && *abort_flag == 0) {
      tc_fence_after();
      float* crow = p.C + (size_t)z * p.c_zstride + (size_t)(m0 + 32 * q + lane) * p.ldc + n0;
      const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
      for (int c = 0; c < kTileMN; c += 16) {
        float v[16];
        tmem_ld16(taddr + c, v);
#pragma unroll
        for (int i = 0; i < 16; i += 4) *reinterpret_cast<float4*>(crow + c + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag != 0) {
    if (threadIdx.x == 0) flag_status(p.status, SAGA_STATUS_TIMEOUT);
    if (warp == 0 && lane == 0)
      for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t)
        mbar_wait_drain(&full[t % kStages], (t / kStages) & 1);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- 3. pseudoinverse per pair
// Pairs (a, b), a < b, in the order (0,1), (0,2), ..., (0,h-1), (1,2), ...
__host__ __device__ inline void pair_of(int p, int h, int* a, int* b) {
  int aa = 0;
  while (p >= h - 1 - aa) {
    p -= h - 1 - aa;
    ++aa;
  }
  *a = aa;
  *b = aa + 1 + p;
}

struct PairParams {
  const float* Sg;  // [h_k][128][128] fp32 Gram blocks S_r (top-left d x d)
  double* V;        // [npairs][d][d] eigenvectors (work, used where they do not fit in shared memory)
  double* A;        // [npairs][d][d] S_a (S_a + S_b)^+
  double* B;        // [npairs][d][d] S_b (S_a + S_b)^+
  int h_k;
  int max_sweeps;
  double rtol;      // eigenvalues at most rtol * max |eigenvalue| count as zero
};

// Shared memory of the pseudoinverse kernel: S, and V where it fits (d = 64),
// rows padded by one element so that column walks do not hit one bank.
__host__ __device__ constexpr int pinv_smem_bytes(int d) { return (d == 64 ? 2 : 1) * d * (d + 1) * 8; }

// One CTA per pair: S = S_a + S_b (fp64, in shared memory) is diagonalised by
// parallel cyclic Jacobi rotations.  Each round rotates the d/2 disjoint index
// pairs of the circle method, all angles computed from the round's start;
// S <- J^T S J is applied one 2 x 2 block (row pair, column pair) per thread
// step (the blocks partition S, so one barrier separates rounds) and V <- V J
// one (row, column pair) per step.  Sweeps stop once the off-diagonal mass is
// below 1e-30 of the total, or after max_sweeps.  Then S^+ = V diag(1/lambda)
// V^T over the eigenvalues above the cut, and A = S_a S^+, B = S_b S^+.
template <int DD, int NT>
__global__ void __launch_bounds__(NT) merge_pinv_kernel(const PairParams p) {
  constexpr int H = DD / 2;
  constexpr bool VSH = DD == 64;  // V beside S in shared memory
  constexpr int LS = DD + 1;                // row stride of S
  constexpr int LV = VSH ? DD + 1 : DD;     // row stride of V
  extern __shared__ double sh[];
  __shared__ double cs[H], sn[H];
  __shared__ int pp[H], qq[H];
  __shared__ double red_off[NT / 32], red_tot[NT / 32];
  __shared__ double inv[DD];
  __shared__ int done;
  __shared__ double lmax;
  const int pair = blockIdx.x, tid = threadIdx.x;
  int a, b;
  pair_of(pair, p.h_k, &a, &b);
  double* S = sh;
  double* V = VSH ? sh + DD * LS : p.V + (size_t)pair * DD * DD;
  const float* Sa = p.Sg + (size_t)a * 128 * 128;
  const float* Sb = p.Sg + (size_t)b * 128 * 128;
  for (int e = tid; e < DD * DD; e += NT) {
    const int i = e / DD, j = e % DD;
    S[i * LS + j] = (double)Sa[i * 128 + j] + (double)Sb[i * 128 + j];
    V[i * LV + j] = i == j ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int sweep = 0; sweep < p.max_sweeps; ++sweep) {
    // convergence: off-diagonal mass against the total
    double off = 0.0, tot = 0.0;
    for (int e = tid; e < DD * DD; e += NT) {
      const int i = e / DD, j = e % DD;
      const double v = S[i * LS + j] * S[i * LS + j];
      tot += v;
      if (i != j) off += v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(0xffffffffu, off, o);
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
    }
    if ((tid & 31) == 0) {
      red_off[tid >> 5] = off;
      red_tot[tid >> 5] = tot;
    }
    __syncthreads();
    if (tid == 0) {
      double o2 = 0.0, t2 = 0.0;
      for (int w = 0; w < NT / 32; ++w) {
        o2 += red_off[w];
        t2 += red_tot[w];
      }
      done = (o2 <= 1e-30 * t2) ? 1 : 0;
    }
    __syncthreads();
    if (done) break;
    for (int r = 0; r < DD - 1; ++r) {
      // round r of the circle method: (r, d-1) and ((r+k) mod (d-1), (r-k) mod (d-1)), k = 1 .. d/2-1
      if (tid < H) {
        int i, j;
        if (tid == 0) {
          i = r;
          j = DD - 1;
        } else {
          i = (r + tid) % (DD - 1);
          j = (r - tid + (DD - 1)) % (DD - 1);
        }
        if (i > j) {
          const int x = i;
          i = j;
          j = x;
        }
        const double apq = S[i * LS + j], app = S[i * LS + i], aqq = S[j * LS + j];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double theta = (aqq - app) / (2.0 * apq);
          const double t = (theta >= 0.0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
          c = 1.0 / sqrt(t * t + 1.0);
          s = t * c;
        }
        cs[tid] = c;
        sn[tid] = s;
        pp[tid] = i;
        qq[tid] = j;
      }
      __syncthreads();
      // S <- J^T S J, block (row pair m, column pair n): rows first, then columns
      for (int e = tid; e < H * H; e += NT) {
        const int m = e / H, n = e % H;
        const int i = pp[m], j = qq[m], k = pp[n], l = qq[n];
        const double cm = cs[m], sm = sn[m], cn = cs[n], snn = sn[n];
        const double xik = S[i * LS + k], xil = S[i * LS + l], xjk = S[j * LS + k], xjl = S[j * LS + l];
        const double yik = cm * xik - sm * xjk, yjk = sm * xik + cm * xjk;
        const double yil = cm * xil - sm * xjl, yjl = sm * xil + cm * xjl;
        S[i * LS + k] = cn * yik - snn * yil;
        S[i * LS + l] = snn * yik + cn * yil;
        S[j * LS + k] = cn * yjk - snn * yjl;
        S[j * LS + l] = snn * yjk + cn * yjl;
      }
      // V <- V J
      for (int e = tid; e < DD * H; e += NT) {
        const int row = e / H, n = e % H;
        const int k = pp[n], l = qq[n];
        const double cn = cs[n], snn = sn[n];
        const double vk = V[row * LV + k], vl = V[row * LV + l];
        V[row * LV + k] = cn * vk - snn * vl;
        V[row * LV + l] = snn * vk + cn * vl;
      }
      __syncthreads();
    }
  }
  // eigenvalues on the diagonal; the cut, then S^+ = V diag(inv) V^T (into shared memory over S)
  if (tid == 0) {
    double mx = 0.0;
    for (int i = 0; i < DD; ++i) mx = fmax(mx, fabs(S[i * LS + i]));
    lmax = mx;
  }
  __syncthreads();
  if (tid < DD) {
    const double l = S[tid * LS + tid];
    inv[tid] = fabs(l) > p.rtol * lmax ? 1.0 / l : 0.0;
  }
  __syncthreads();
  for (int e = tid; e < DD * DD; e += NT) {
    const int i = e / DD, j = e % DD;
    double acc = 0.0;
    for (int k = 0; k < DD; ++k) acc += V[i * LV + k] * inv[k] * V[j * LV + k];
    S[i * LS + j] = acc;
  }
  __syncthreads();
  double* A = p.A + (size_t)pair * DD * DD;
  double* B = p.B + (size_t)pair * DD * DD;
  for (int e = tid; e < DD * DD; e += NT) {
    const int i = e / DD, j = e % DD;
    double x = 0.0, y = 0.0;
    for (int k = 0; k < DD; ++k) {
      x += (double)Sa[i * 128 + k] * S[k * LS + j];
      y += (double)Sb[i * 128 + k] * S[k * LS + j];
    }
    A[e] = x;
    B[e] = y;
  }
}

// ---------------------------------------------------------------- 4. loss terms
// Eq. 13 through the Gram matrices: for pair (a, b) and head r in {a, b},
// with D_r = M(a, b) - W_r, the term is tr(D_r^T G D_r S_r) =
// sum_{i, c} (G D_r)[i][c] (D_r S_r)[i][c].  Since M(a, b) = W_a A + W_b B,
// G D_r = (GW_a A + GW_b B) - GW_r with GW_r = G W_r computed once per head;
// that leaves per pair two (D x 2d) x (2d x d) products and two D x d x d ones
// instead of a D x D x d product per pair and head.  All sums in fp64.
//
// Thread tile of both kernels: 4 rows (4 ty .. 4 ty + 3 of a 64-row block) by
// DD / 16 columns (tx, tx + 16, ...), 256 threads.
constexpr int kRows = 64;  // rows per CTA
constexpr int kKc = 16;    // k-chunk staged in shared memory

struct GwParams {
  const float* G;  // [Dp][Dp] (ld = ldg)
  long long ldg;
  const float* W;  // [h_k][D][d]
  double* GW;      // [h_k][D][d]
  int D;
};

constexpr int kGwRows = 128;  // rows of G W_r per CTA (8 per thread)
constexpr int kGwKc = 32;     // k-chunk of the G W_r product
constexpr int kGwLd = kGwKc + 4;  // padded row of the staged G chunk (16-byte rows, no common bank)

// Two buffers of raw fp32 chunks: G [kGwRows][kGwLd] and W_r [kGwKc][DD].
template <int DD>
__host__ __device__ constexpr int gw_smem_bytes() { return 2 * (kGwRows * kGwLd + kGwKc * DD) * 4; }

// GW_r = G W_r: grid (row blocks of 128, h_k); thread tile 8 rows (8 ty .. 8 ty + 7)
// by DD / 16 columns (tx, tx + 16, ...).  The next k-chunk is copied into the
// other buffer by cp.async while the current one is multiplied.
template <int DD>
__global__ void __launch_bounds__(256) merge_gw_kernel(const GwParams p) {
  constexpr int CT = DD / 16;
  extern __shared__ __align__(16) float gsf[];
  float* Gs = gsf;                          // [2][kGwRows][kGwLd]
  float* Ws = gsf + 2 * kGwRows * kGwLd;    // [2][kGwKc][DD]
  const int r = blockIdx.y, i0 = blockIdx.x * kGwRows, tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const float* Wr = p.W + (size_t)r * p.D * DD;
  // rows i0 .. i0 + 127 and columns below the padded size are inside G (zero past D)
  auto issue = [&](int k0, int buf) {
    float* gd = Gs + buf * kGwRows * kGwLd;
    for (int c = tid; c < kGwRows * (kGwKc / 4); c += 256) {
      const int rr = c / (kGwKc / 4), q4 = c % (kGwKc / 4);
      cp_async16(gd + rr * kGwLd + q4 * 4, p.G + (size_t)(i0 + rr) * p.ldg + k0 + q4 * 4);
    }
    float* wd = Ws + buf * kGwKc * DD;
    for (int c = tid; c < kGwKc * (DD / 4); c += 256) {
      const int kk = c / (DD / 4), q4 = c % (DD / 4), gk = k0 + kk;
      cp_async16_zfill(wd + kk * DD + q4 * 4, Wr + (size_t)(gk < p.D ? gk : 0) * DD + q4 * 4, gk < p.D);
    }
    cp_async_commit();
  };
  double acc[8][CT];
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int c = 0; c < CT; ++c) acc[q][c] = 0.0;
  issue(0, 0);
  int buf = 0;
  for (int k0 = 0; k0 < p.D; k0 += kGwKc, buf ^= 1) {
    const bool more = k0 + kGwKc < p.D;
    if (more) {
      issue(k0 + kGwKc, buf ^ 1);
      cp_async_wait_one();
    } else {
      cp_async_wait_all();
    }
    __syncthreads();
    const float* gs = Gs + buf * kGwRows * kGwLd;
    const float* ws = Ws + buf * kGwKc * DD;
#pragma unroll 4
    for (int kk = 0; kk < kGwKc; ++kk) {
      double g[8], w[CT];
#pragma unroll
      for (int q = 0; q < 8; ++q) g[q] = (double)gs[(8 * ty + q) * kGwLd + kk];
#pragma unroll
      for (int c = 0; c < CT; ++c) w[c] = (double)ws[kk * DD + tx + 16 * c];
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int c = 0; c < CT; ++c) acc[q][c] = fma(g[q], w[c], acc[q][c]);
    }
    __syncthreads();  // this buffer is refilled two chunks on
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int gi = i0 + 8 * ty + q;
    if (gi < p.D)
#pragma unroll
      for (int c = 0; c < CT; ++c) p.GW[((size_t)r * p.D + gi) * DD + tx + 16 * c] = acc[q][c];
  }
}

struct LossParams {
  const float* W;     // [h_k][D][d]
  const double* GW;   // [h_k][D][d]
  const double* A;    // [npairs][d][d]
  const double* B;    // [npairs][d][d]
  const float* Sg;    // [h_k][128][128]
  double* M;          // [npairs][D][d] (written)
  double* partial;    // [npairs][nblk] (written)
  int D, h_k, nblk;
};

template <int DD>
struct LossSmem {
  // phase 1, two buffers of raw k-chunks: A and B rows (fp64), the block's
  // W_a and W_b columns (fp32) and GW_a and GW_b columns (fp64)
  static constexpr int AB = 2 * kKc * DD * 8;
  static constexpr int XW = 2 * kRows * kKc * 4;
  static constexpr int YW = 2 * kRows * kKc * 8;
  static constexpr int BUF = AB + XW + YW;
  static constexpr int P1 = 2 * BUF;
  // phase 2: M rows (fp64), W_r rows and S_r (fp32)
  static constexpr int M_OFF = 0;
  static constexpr int W_OFF = kRows * DD * 8;
  static constexpr int S_OFF = W_OFF + kRows * DD * 4;
  static constexpr int P2 = S_OFF + DD * DD * 4;
  static constexpr int BYTES = P1 > P2 ? P1 : P2;
};

// Merged projections and the pair's loss over one 64-row block: grid (row blocks, pairs).
template <int DD>
__global__ void __launch_bounds__(256) merge_loss_kernel(const LossParams p) {
  using SM = LossSmem<DD>;
  constexpr int CT = DD / 16;
  extern __shared__ double lsh[];
  __shared__ double red[8];
  const int blk = blockIdx.x, pair = blockIdx.y, tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const int i0 = blk * kRows;
  int a, b;
  pair_of(pair, p.h_k, &a, &b);
  const double* A = p.A + (size_t)pair * DD * DD;
  const double* B = p.B + (size_t)pair * DD * DD;
  const float* Wa = p.W + (size_t)a * p.D * DD;
  const float* Wb = p.W + (size_t)b * p.D * DD;
  const double* GWa = p.GW + (size_t)a * p.D * DD;
  const double* GWb = p.GW + (size_t)b * p.D * DD;
  // phase 1: M = W_a A + W_b B and GM = GW_a A + GW_b B for this thread's rows and columns
  double m[4][CT], gm[4][CT];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int c = 0; c < CT; ++c) m[q][c] = gm[q][c] = 0.0;
  {
    uint8_t* base = reinterpret_cast<uint8_t*>(lsh);
    auto issue = [&](int k0, int buf) {
      uint8_t* bb = base + buf * SM::BUF;
      double* As = reinterpret_cast<double*>(bb);  // [kKc][DD], then Bs
      float* Xa = reinterpret_cast<float*>(bb + SM::AB);  // [kRows][kKc], then Xb
      double* Ya = reinterpret_cast<double*>(bb + SM::AB + SM::XW);  // [kRows][kKc], then Yb
      for (int c = tid; c < kKc * DD / 2; c += 256) {
        cp_async16(As + 2 * c, A + (size_t)k0 * DD + 2 * c);
        cp_async16(As + kKc * DD + 2 * c, B + (size_t)k0 * DD + 2 * c);
      }
      for (int c = tid; c < kRows * (kKc / 4); c += 256) {
        const int rr = c / (kKc / 4), q4 = c % (kKc / 4), gi = i0 + rr;
        const size_t o = (size_t)(gi < p.D ? gi : 0) * DD + k0 + q4 * 4;
        cp_async16_zfill(Xa + rr * kKc + q4 * 4, Wa + o, gi < p.D);
        cp_async16_zfill(Xa + kRows * kKc + rr * kKc + q4 * 4, Wb + o, gi < p.D);
      }
      for (int c = tid; c < kRows * (kKc / 2); c += 256) {
        const int rr = c / (kKc / 2), q2 = c % (kKc / 2), gi = i0 + rr;
        const size_t o = (size_t)(gi < p.D ? gi : 0) * DD + k0 + q2 * 2;
        cp_async16_zfill(Ya + rr * kKc + q2 * 2, GWa + o, gi < p.D);
        cp_async16_zfill(Ya + kRows * kKc + rr * kKc + q2 * 2, GWb + o, gi < p.D);
      }
      cp_async_commit();
    };
    issue(0, 0);
    int buf = 0;
    for (int k0 = 0; k0 < DD; k0 += kKc, buf ^= 1) {
      const bool more = k0 + kKc < DD;
      if (more) {
        issue(k0 + kKc, buf ^ 1);
        cp_async_wait_one();
      } else {
        cp_async_wait_all();
      }
      __syncthreads();
      const uint8_t* bb = base + buf * SM::BUF;
      const double* As = reinterpret_cast<const double*>(bb);
      const double* Bs = As + kKc * DD;
      const float* Xa = reinterpret_cast<const float*>(bb + SM::AB);
      const float* Xb = Xa + kRows * kKc;
      const double* Ya = reinterpret_cast<const double*>(bb + SM::AB + SM::XW);
      const double* Yb = Ya + kRows * kKc;
#pragma unroll 2
      for (int kk = 0; kk < kKc; ++kk) {
        double av[CT], bv[CT];
#pragma unroll
        for (int c = 0; c < CT; ++c) {
          av[c] = As[kk * DD + tx + 16 * c];
          bv[c] = Bs[kk * DD + tx + 16 * c];
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int rr = 4 * ty + q;
          const double xa = (double)Xa[rr * kKc + kk], xb = (double)Xb[rr * kKc + kk];
          const double ya = Ya[rr * kKc + kk], yb = Yb[rr * kKc + kk];
#pragma unroll
          for (int c = 0; c < CT; ++c) {
            m[q][c] = fma(xa, av[c], fma(xb, bv[c], m[q][c]));
            gm[q][c] = fma(ya, av[c], fma(yb, bv[c], gm[q][c]));
          }
        }
      }
      __syncthreads();  // this buffer is refilled two chunks on
    }
  }
  // phase 2: M rows to global and shared memory; then for r in {a, b}: (M - W_r) S_r against GM - GW_r
  double* Ms = reinterpret_cast<double*>(reinterpret_cast<char*>(lsh) + SM::M_OFF);  // [kRows][DD]
  float* Wsm = reinterpret_cast<float*>(reinterpret_cast<char*>(lsh) + SM::W_OFF);  // [kRows][DD]
  float* Ss = reinterpret_cast<float*>(reinterpret_cast<char*>(lsh) + SM::S_OFF);   // [DD][DD]
  double* Mout = p.M + (size_t)pair * p.D * DD;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int rr = 4 * ty + q, gi = i0 + rr;
#pragma unroll
    for (int c = 0; c < CT; ++c) {
      Ms[rr * DD + tx + 16 * c] = m[q][c];
      if (gi < p.D) Mout[(size_t)gi * DD + tx + 16 * c] = m[q][c];
    }
  }
  double part = 0.0;
  for (int side = 0; side < 2; ++side) {
    const int r = side == 0 ? a : b;
    const float* Wr = side == 0 ? Wa : Wb;
    const double* GWr = side == 0 ? GWa : GWb;
    const float* Sr = p.Sg + (size_t)r * 128 * 128;
    __syncthreads();  // Ms written / the previous side is done with Wsm and Ss
    for (int e = tid; e < kRows * DD; e += 256) {
      const int rr = e / DD, c = e % DD, gi = i0 + rr;
      Wsm[e] = gi < p.D ? Wr[(size_t)gi * DD + c] : 0.f;
    }
    for (int e = tid; e < DD * DD; e += 256) Ss[e] = Sr[(e / DD) * 128 + (e % DD)];
    __syncthreads();
    double ds[4][CT];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int c = 0; c < CT; ++c) ds[q][c] = 0.0;
#pragma unroll 2
    for (int k = 0; k < DD; ++k) {
      double sv[CT];
#pragma unroll
      for (int c = 0; c < CT; ++c) sv[c] = (double)Ss[k * DD + tx + 16 * c];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int rr = 4 * ty + q;
        const double dk = Ms[rr * DD + k] - (double)Wsm[rr * DD + k];
#pragma unroll
        for (int c = 0; c < CT; ++c) ds[q][c] = fma(dk, sv[c], ds[q][c]);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int gi = i0 + 4 * ty + q;
      if (gi < p.D)
#pragma unroll
        for (int c = 0; c < CT; ++c) part += (gm[q][c] - GWr[(size_t)gi * DD + tx + 16 * c]) * ds[q][c];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((tid & 31) == 0) red[tid >> 5] = part;
  __syncthreads();
  if (tid == 0) {
    double s = 0.0;
    for (int w = 0; w < 8; ++w) s += red[w];
    p.partial[(size_t)pair * p.nblk + blk] = s;
  }
}

// ---------------------------------------------------------------- 5. matching
// w(a, b) = sum of the pair's loss terms (fixed order).  Every perfect
// matching of the h_k heads has an index: pairing the lowest unmatched head
// with the c-th remaining one at each level, c taken as mixed-radix digits
// (most significant first), so indices follow the order of the usual
// recursive enumeration.  Each thread scores a range of indices; the lowest
// total wins (ties: the lowest index).
struct MatchParams {
  const double* partial;  // [npairs][nblk]
  const double* M;        // [npairs][D][d]
  float* pair_loss;       // [h_k][h_k]
  int* pairing;           // [h_k]
  float* merged;          // [h_k / 2][D][d]
  int h_k, npairs, nblk, D, d;
};

__device__ inline long long double_factorial_odd(int n) {  // (n-1)!! for even n: number of perfect matchings
  long long v = 1;
  for (int k = n - 1; k > 1; k -= 2) v *= k;
  return v;
}

__global__ void __launch_bounds__(1024) merge_match_kernel(const MatchParams p) {
  __shared__ double w[kMaxHeads][kMaxHeads];
  __shared__ double best_total[1024 / 32];
  __shared__ long long best_index[1024 / 32];
  __shared__ int partner[kMaxHeads];
  const int h = p.h_k, tid = threadIdx.x;
  for (int e = tid; e < h * h; e += blockDim.x) w[e / h][e % h] = 0.0;
  __syncthreads();
  for (int pr = tid; pr < p.npairs; pr += blockDim.x) {
    int a, b;
    pair_of(pr, h, &a, &b);
    double s = 0.0;
    for (int k = 0; k < p.nblk; ++k) s += p.partial[(size_t)pr * p.nblk + k];
    w[a][b] = w[b][a] = s;
  }
  __syncthreads();
  for (int e = tid; e < h * h; e += blockDim.x) p.pair_loss[e] = (float)w[e / h][e % h];
  const long long count = double_factorial_odd(h);
  double my_best = INFINITY;
  long long my_idx = -1;
  for (long long idx = tid; idx < count; idx += blockDim.x) {
    int rem[kMaxHeads];
    int n = h;
    for (int i = 0; i < h; ++i) rem[i] = i;
    long long x = idx, radix_prod = count;
    double total = 0.0;
    while (n > 0) {
      radix_prod /= (n - 1);  // matchings of the n - 2 heads left after this level
      const int c = (int)(x / radix_prod);
      x -= (long long)c * radix_prod;
      const int a = rem[0], b = rem[1 + c];
      total += w[a][b];
      for (int i = 1 + c; i < n - 1; ++i) rem[i] = rem[i + 1];  // drop b
      for (int i = 0; i < n - 2; ++i) rem[i] = rem[i + 1];      // drop a
      n -= 2;
    }
    if (total < my_best) {  // indices rise within a thread: a later tie never replaces
      my_best = total;
      my_idx = idx;
    }
  }
  // block argmin (lowest total, then lowest index)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ot = __shfl_xor_sync(0xffffffffu, my_best, o);
    const long long oi = __shfl_xor_sync(0xffffffffu, my_idx, o);
    if (ot < my_best || (ot == my_best && oi >= 0 && (my_idx < 0 || oi < my_idx))) {
      my_best = ot;
      my_idx = oi;
    }
  }
  if ((tid & 31) == 0) {
    best_total[tid >> 5] = my_best;
    best_index[tid >> 5] = my_idx;
  }
  __syncthreads();
  if (tid == 0) {
    double bt = INFINITY;
    long long bi = -1;
    for (int w2 = 0; w2 < (int)(blockDim.x / 32); ++w2)
      if (best_index[w2] >= 0 && (best_total[w2] < bt || (best_total[w2] == bt && best_index[w2] < bi))) {
        bt = best_total[w2];
        bi = best_index[w2];
      }
    // decode the winning index
    int rem[kMaxHeads];
    int n = h;
    for (int i = 0; i < h; ++i) rem[i] = i;
    long long x = bi, radix_prod = count;
    while (n > 0) {
      radix_prod /= (n - 1);
      const int c = (int)(x / radix_prod);
      x -= (long long)c * radix_prod;
      const int a = rem[0], b = rem[1 + c];
      partner[a] = b;
      partner[b] = a;
      for (int i = 1 + c; i < n - 1; ++i) rem[i] = rem[i + 1];
      for (int i = 0; i < n - 2; ++i) rem[i] = rem[i + 1];
      n -= 2;
    }
    for (int i = 0; i < h; ++i) p.pairing[i] = partner[i];
  }
}

// The merged projections of the chosen pairs as fp32, pairs ordered by their
// smaller head: grid (ceil(D d / 1024), h_k / 2), one element per thread.
__global__ void __launch_bounds__(1024) merge_emit_kernel(const MatchParams p) {
  const int slot = blockIdx.y;
  int a = 0, seen = -1, b = 0;
  for (; a < p.h_k; ++a) {
    b = p.pairing[a];
    if (b > a && ++seen == slot) break;
  }
  if (a >= p.h_k) return;
  int pr = 0;
  for (int x = 0; x < a; ++x) pr += p.h_k - 1 - x;
  pr += b - a - 1;
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e < (long long)p.D * p.d)
    p.merged[(size_t)slot * p.D * p.d + e] = (float)p.M[(size_t)pr * p.D * p.d + e];
}

}  // namespace merge
}  // namespace saga

// ================================================================ host
using namespace saga::merge;

namespace {

thread_local char g_merge_err[256] = "";

int merge_fail(int code, const char* msg) {
  snprintf(g_merge_err, sizeof(g_merge_err), "%s", msg);
  return code;
}

struct MergeLayout {
  long long Dp, Tp, Kq;
  size_t status, xt, qt, g, sg, v, a, b, gw, m, partial, total;
  int npairs, nblk;
};

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

MergeLayout merge_layout(const saga_merge_shape* s) {
  MergeLayout L{};
  const int g = s->h_q / s->h_k;
  L.Dp = round_up(s->hidden, kTileMN);
  L.Tp = round_up(s->tokens, kTileK);
  L.Kq = round_up((long long)g * s->tokens, kTileK);
  L.npairs = s->h_k * (s->h_k - 1) / 2;
  L.nblk = (s->hidden + kRows - 1) / kRows;
  size_t off = 0;
  L.status = off;
  off = a256(off + 16);
  L.xt = off;
  off = a256(off + (size_t)L.Dp * L.Tp * 2);
  L.qt = off;
  off = a256(off + (size_t)s->h_k * kTileMN * L.Kq * 2);
  L.g = off;
  off = a256(off + (size_t)L.Dp * L.Dp * 4);
  L.sg = off;
  off = a256(off + (size_t)s->h_k * kTileMN * kTileMN * 4);
  L.v = off;
  off = a256(off + (size_t)L.npairs * s->d * s->d * 8);
  L.a = off;
  off = a256(off + (size_t)L.npairs * s->d * s->d * 8);
  L.b = off;
  off = a256(off + (size_t)L.npairs * s->d * s->d * 8);
  L.gw = off;
  off = a256(off + (size_t)s->h_k * s->hidden * s->d * 8);
  L.m = off;
  off = a256(off + (size_t)L.npairs * s->hidden * s->d * 8);
  L.partial = off;
  off = a256(off + (size_t)L.npairs * L.nblk * 8);
  L.total = off;
  return L;
}

int merge_validate(const saga_merge_shape* s) {
  if (s == nullptr) return merge_fail(SAGA_ERR_ARG, "shape is NULL");
  if (s->tokens < 1 || s->hidden < 1 || s->h_q < 1 || s->h_k < 2)
    return merge_fail(SAGA_ERR_ARG, "tokens, hidden, h_q must be >= 1 and h_k >= 2");
  if (s->d != 64 && s->d != 128) return merge_fail(SAGA_ERR_UNSUPPORTED, "head dim must be 64 or 128");
  if (s->h_k % 2 != 0 || s->h_k > kMaxHeads)
    return merge_fail(SAGA_ERR_UNSUPPORTED, "h_k must be even and at most 16 (pairs, matched exhaustively)");
  if (s->h_q % s->h_k != 0) return merge_fail(SAGA_ERR_ARG, "h_q must be a multiple of h_k");
  if ((long long)s->tokens * s->h_q > (1ll << 30) || (long long)s->hidden > (1 << 20) ||
      (long long)s->tokens * s->hidden > (1ll << 31))
    return merge_fail(SAGA_ERR_UNSUPPORTED, "problem too large for 32-bit indexing");
  return SAGA_OK;
}

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn merge_encoder() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(ptr);
  });
  return fn;
}

// bf16 [rows, cols] row-major (cols contiguous, a multiple of 64): boxes of 64 columns x 128 rows,
// 128-byte swizzle (the K-major operand layout of the MMA)
int operand_map(CUtensorMap* m, const void* base, long long rows, long long cols) {
  EncodeFn enc = merge_encoder();
  if (enc == nullptr) return merge_fail(SAGA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable from the driver");
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kTileK, (cuuint32_t)kTileMN};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return merge_fail(SAGA_ERR_CUDA, "cuTensorMapEncodeTiled failed (merge operand)");
  return SAGA_OK;
}

int cuda_err(cudaError_t e, const char* what) {
  snprintf(g_merge_err, sizeof(g_merge_err), "%s: %s", what, cudaGetErrorString(e));
  return SAGA_ERR_CUDA;
}

std::atomic<uint64_t> g_smem_set{0};

}  // namespace

extern "C" {

size_t saga_merge_workspace_bytes(const saga_merge_shape* s) {
  if (merge_validate(s)) return 0;
  return merge_layout(s).total;
}

const char* saga_merge_last_error(void) { return g_merge_err; }

int saga_key_head_merge(const saga_merge_shape* s, const void* x, const void* q, const float* w_k, float* pair_loss,
                        int* pairing, float* w_k_merged, void* workspace, size_t ws_bytes, void* stream) {
  g_merge_err[0] = '\0';
  int rc = merge_validate(s);
  if (rc) return rc;
  if (!x || !q || !w_k || !pair_loss || !pairing || !w_k_merged) return merge_fail(SAGA_ERR_ARG, "NULL pointer");
  const uintptr_t al = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(q) |
                       reinterpret_cast<uintptr_t>(w_k) | reinterpret_cast<uintptr_t>(w_k_merged);
  if (al & 15u) return merge_fail(SAGA_ERR_ARG, "x, q, w_k and w_k_merged must be 16-byte aligned");
  const MergeLayout L = merge_layout(s);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return merge_fail(SAGA_ERR_WORKSPACE, "workspace NULL or not 256-byte aligned");
  if (ws_bytes < L.total) return merge_fail(SAGA_ERR_WORKSPACE, "workspace smaller than saga_merge_workspace_bytes");
  char* base = static_cast<char*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint16_t* xt = reinterpret_cast<uint16_t*>(base + L.xt);
  uint16_t* qt = reinterpret_cast<uint16_t*>(base + L.qt);
  float* G = reinterpret_cast<float*>(base + L.g);
  float* Sg = reinterpret_cast<float*>(base + L.sg);
  unsigned* status = reinterpret_cast<unsigned*>(base + L.status);
  CUtensorMap mx, mq;
  rc = operand_map(&mx, xt, L.Dp, L.Tp);
  if (rc) return rc;
  rc = operand_map(&mq, qt, (long long)s->h_k * kTileMN, L.Kq);
  if (rc) return rc;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_err(e, "cudaGetDevice");
  const uint64_t bit = 1ull << (dev & 63);
  if (!(g_smem_set.load() & bit)) {
    e = cudaFuncSetAttribute(merge_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmSmem::ALLOC);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(merge_pinv_kernel<64, 1024>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               pinv_smem_bytes(64));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(merge_pinv_kernel<128, 1024>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               pinv_smem_bytes(128));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(merge_gw_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, gw_smem_bytes<64>());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(merge_gw_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               gw_smem_bytes<128>());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(merge_loss_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               LossSmem<64>::BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(merge_loss_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               LossSmem<128>::BYTES);
    if (e != cudaSuccess) return cuda_err(e, "cudaFuncSetAttribute");
    g_smem_set.fetch_or(bit);
  }
  const int g = s->h_q / s->h_k;
  // everything validated: enqueue
  e = cudaMemsetAsync(base, 0, L.sg, st);  // status, the padded transposes and G
  if (e != cudaSuccess) return cuda_err(e, "cudaMemsetAsync");
  const dim3 tb(32, 8);
  merge_transpose_kernel<<<dim3((s->hidden + 31) / 32, (s->tokens + 31) / 32, 1), tb, 0, st>>>(
      static_cast<const uint16_t*>(x), s->tokens, s->hidden, s->hidden, 0, xt, L.Tp, 1, 0, 0);
  merge_transpose_kernel<<<dim3((s->d + 31) / 32, (s->tokens + 31) / 32, s->h_q), tb, 0, st>>>(
      static_cast<const uint16_t*>(q), s->tokens, s->d, (long long)s->h_q * s->d, s->d, qt, L.Kq, g,
      (long long)kTileMN * L.Kq, s->tokens);
  GemmParams gp{};
  gp.Mz = gp.Nz = (int)L.Dp;
  gp.k_blocks = (int)(L.Tp / kTileK);
  gp.ldc = L.Dp;
  gp.c_zstride = 0;
  gp.C = G;
  gp.status = status;
  merge_gemm_kernel<<<dim3((unsigned)(L.Dp / kTileMN), (unsigned)(L.Dp / kTileMN), 1), 192, GemmSmem::ALLOC, st>>>(
      mx, mx, gp);
  gp.Mz = gp.Nz = kTileMN;
  gp.k_blocks = (int)(L.Kq / kTileK);
  gp.ldc = kTileMN;
  gp.c_zstride = (long long)kTileMN * kTileMN;
  gp.C = Sg;
  merge_gemm_kernel<<<dim3(1, 1, s->h_k), 192, GemmSmem::ALLOC, st>>>(mq, mq, gp);
  PairParams pp{};
  pp.Sg = Sg;
  pp.V = reinterpret_cast<double*>(base + L.v);
  pp.A = reinterpret_cast<double*>(base + L.a);
  pp.B = reinterpret_cast<double*>(base + L.b);
  pp.h_k = s->h_k;
  pp.max_sweeps = 30;
  pp.rtol = 1e-5;  // the Gram matrices carry fp32 rounding: smaller eigenvalues are noise
  if (s->d == 64)
    merge_pinv_kernel<64, 1024><<<L.npairs, 1024, pinv_smem_bytes(64), st>>>(pp);
  else
    merge_pinv_kernel<128, 1024><<<L.npairs, 1024, pinv_smem_bytes(128), st>>>(pp);
  GwParams gw{};
  gw.G = G;
  gw.ldg = L.Dp;
  gw.W = w_k;
  gw.GW = reinterpret_cast<double*>(base + L.gw);
  gw.D = s->hidden;
  const dim3 ggrid((unsigned)((s->hidden + kGwRows - 1) / kGwRows), (unsigned)s->h_k);
  if (s->d == 64)
    merge_gw_kernel<64><<<ggrid, 256, gw_smem_bytes<64>(), st>>>(gw);
  else
    merge_gw_kernel<128><<<ggrid, 256, gw_smem_bytes<128>(), st>>>(gw);
  LossParams lp{};
  lp.W = w_k;
  lp.GW = gw.GW;
  lp.A = pp.A;
  lp.B = pp.B;
  lp.Sg = Sg;
  lp.M = reinterpret_cast<double*>(base + L.m);
  lp.partial = reinterpret_cast<double*>(base + L.partial);
  lp.D = s->hidden;
  lp.h_k = s->h_k;
  lp.nblk = L.nblk;
  const dim3 lgrid((unsigned)L.nblk, (unsigned)L.npairs);
  if (s->d == 64)
    merge_loss_kernel<64><<<lgrid, 256, LossSmem<64>::BYTES, st>>>(lp);
  else
    merge_loss_kernel<128><<<lgrid, 256, LossSmem<128>::BYTES, st>>>(lp);
  MatchParams mp{};
  mp.partial = lp.partial;
  mp.M = lp.M;
  mp.pair_loss = pair_loss;
  mp.pairing = pairing;
  mp.merged = w_k_merged;
  mp.h_k = s->h_k;
  mp.npairs = L.npairs;
  mp.nblk = L.nblk;
  mp.D = s->hidden;
  mp.d = s->d;
  merge_match_kernel<<<1, 1024, 0, st>>>(mp);
  merge_emit_kernel<<<dim3((unsigned)(((long long)s->hidden * s->d + 1023) / 1024), (unsigned)(s->h_k / 2)), 1024, 0,
                      st>>>(mp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_err(e, "merge launch");
  return SAGA_OK;
}

}  // extern "C"
