// bsa_backward.cu -- the backward pass of block-sparse attention (dQ, dK, dV).
//
// "Block Sparse Attention with Log-Linear Complexity" notes that the sparse
// product falls back to dense work in the backward pass (section 4.2) and
// trains with the pattern (section 5.3).  With the forward's O and LSE saved,
// per (b, h), query q and allowed key k (the block row's blocks, token-level
// causal mask when asked):
//   P = exp(scale q.k - LSE_q),  D_q = dO_q . O_q,
//   dV_k = sum_q P dO_q,  dS = P (dO_q . v_k - D_q),
//   dQ_q = scale sum_k dS k_k,  dK_k = scale sum_q dS q_q.
// Three kernels, all on tcgen05 with TMEM accumulators and TMA loads:
//   dot_kernel   D_q = dO_q . O_q for every query row (HBM-bound, CUDA cores);
//   dkdv_kernel  one CTA per 128-key tile of one (b, h): walks the union of
//                the query blocks that list the tile's key blocks (from the
//                column-major copy of the CSR), 128 queries a step:
//                  S^T = K Q^T and dP^T = V dO^T      (both operands K-major)
//                  P^T, dS^T in registers, written back to TMEM as bf16
//                  dV += P^T dO and dK += dS^T Q       (A from TMEM, B MN-major)
//   dq_kernel    one CTA per 128-query tile: walks the union of the tile's
//                block rows' columns (the CSR), 128 keys a step:
//                  S = Q K^T and dP = dO V^T; dS to TMEM; dQ += dS K.
// Every output row is produced by exactly one CTA: no atomics, no scratch
// beyond D.  Inside a CTA (8 warps: two per TMEM lane quadrant, one per half
// of the 128 columns) a step runs its MMAs and its elementwise pass in turn
// while the TMA gather of the next step is already in flight (two buffers).
// Every wait is bounded; a wait that gives up sets BSA_STATUS_TIMEOUT and the
// CTA finishes without writing its tile.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstddef>
#include <cstdint>
#include <mutex>

#include "bsa.h"
#include "sm100_ptx.cuh"

namespace bsa {
namespace bwd {

constexpr int kMaxM = 4096;
constexpr int kWords = kMaxM / 32;
constexpr int kThreads = 256;  // two warps per TMEM lane quadrant: one per column half
constexpr long long kWaitLimitCycles = 4000000000LL;  // ~2 s at 1.97 GHz
constexpr float kLog2e = 1.4426950408889634f;

__device__ unsigned int g_bwd_status;

template <int BS, int D>
struct Cfg {
  static constexpr int R = 128 / BS;                 // blocks per 128-row tile
  static constexpr int KATOMS = D / 64;              // 128-byte atoms of a row
  static constexpr int TILE = 128 * D * 2;           // one 128-row bf16 tile
  static constexpr int ATOM = 128 * 128;             // one atom column of a tile
  static constexpr int TMEM_A = 0;                   // S (or S^T): 128 columns
  static constexpr int TMEM_B = 128;                 // dP (or dP^T): 128 columns
  static constexpr int TMEM_C = 256;                 // dV or dQ accumulator: D columns
  static constexpr int TMEM_D = 256 + D;             // dK accumulator: D columns
  static_assert(256 + 2 * D <= 512, "TMEM budget");
};

struct Ctrl {
  uint64_t kv_bar;    // the CTA's own tile (K, V or Q, dO) landed
  uint64_t ld_bar[2]; // the gathered tiles of buffer 0 / 1 landed
  uint64_t mma_bar;   // the step's first two MMAs completed
  uint64_t mma2_bar;  // the step's accumulating MMAs completed
  uint64_t final_bar; // every MMA issued by the CTA completed (teardown)
  uint32_t tmem_base;
  volatile int abort;
  int n_steps;
  int blk[2][4];                    // each buffer's blocks (-1: padding)
  alignas(16) float lse2[128];      // dK/dV: the step's queries' LSE * log2(e)
  alignas(16) float dd[128];        // dK/dV: the step's queries' D
  uint32_t map[4][kWords];          // per tile block: the other side's blocks
  uint32_t uni[kWords];             // union of map[*]
};

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  long long t0 = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 1023u) == 0) {
      if (*abort) return false;
      const long long now = clock64();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kWaitLimitCycles) {
        *abort = 1;
        atomicOr(&g_bwd_status, BSA_STATUS_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  for (uint32_t it = 0; !mbar_try_wait(bar, parity); ++it) {
    if ((it & 1023u) == 1023u && clock64() - t0 > kWaitLimitCycles) {
      atomicOr(&g_bwd_status, BSA_STATUS_TIMEOUT);
      return;
    }
  }
}

struct Args {
  const float* LSE;
  const float* Dq;          // D_q, fp32 [B*H*N]
  const int32_t* ptr;       // row_ptr (dq) or col_ptr (dkdv)
  const int32_t* idx;       // col_idx (dq) or row_idx (dkdv)
  __nv_bfloat16* out0;      // dQ (dq) or dV (dkdv)
  __nv_bfloat16* out1;      // dK (dkdv)
  const int* order;         // tile processed by CTA x: order[x] (heaviest first)
  int H, N, M;
  float scale, scale_log2;
  int causal;
};

// ------------------------------------------------------------ D = dO . O
__global__ void dot_kernel(const __nv_bfloat16* __restrict__ O, const __nv_bfloat16* __restrict__ dO,
                           float* __restrict__ Dq, long long rows, int d) {
  const int lanes_per_row = d / 8;  // 16 bytes per lane
  const int rows_per_warp = 32 / lanes_per_row;
  const int lane = threadIdx.x & 31;
  const int sub = lane / lanes_per_row, part = lane % lanes_per_row;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long r0 = warp * rows_per_warp; r0 < rows; r0 += nwarps * rows_per_warp) {
    const long long r = r0 + sub;
    float acc = 0.f;
    if (r < rows) {
      const uint4 a = reinterpret_cast<const uint4*>(O + r * d)[part];
      const uint4 b = reinterpret_cast<const uint4*>(dO + r * d)[part];
      const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = fmaf(__uint_as_float(av[e] << 16), __uint_as_float(bv[e] << 16), acc);
        acc = fmaf(__uint_as_float(av[e] & 0xffff0000u), __uint_as_float(bv[e] & 0xffff0000u), acc);
      }
    }
    for (int o = lanes_per_row / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (r < rows && part == 0) Dq[r] = acc;
  }
}

// --------------------------------------------------- heavy-first tile order
// The cost of a tile is the total length of its R blocks' lists (an upper
// bound of the union it walks).  Tiles whose blocks appear in long lists (a
// global row or column) take many more steps than the rest; launched in
// plain index order they would start late and leave a long tail, so the
// tile kernels take their tiles heaviest first.
constexpr int kCostBins = 4096;

__global__ void tile_cost_kernel(const int32_t* __restrict__ ptr_a, const int32_t* __restrict__ ptr_b,
                                 int H, int M, int R, int tiles_per_bh, long long T,
                                 int* __restrict__ cost) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const long long bh = t / tiles_per_bh;
  const int tile = static_cast<int>(t - bh * tiles_per_bh);
  const long long base = static_cast<long long>(bh % H) * M + static_cast<long long>(tile) * R;
  int ca = 0, cb = 0;
  for (int r = 0; r < R; ++r) {
    ca += max(0, ptr_a[base + r + 1] - ptr_a[base + r]);
    cb += max(0, ptr_b[base + r + 1] - ptr_b[base + r]);
  }
  cost[t] = min(ca, kCostBins - 1);
  cost[T + t] = min(cb, kCostBins - 1);
}

// Block x of the grid (x = 0, 1) orders the tiles of cost[x*T .. x*T+T) into
// order[x*T ..]: by a counting sort on descending cost (ties in any order)
// when the heaviest tile costs more than twice the mean, or when the launch
// is a few waves (T < few_waves tiles) and the last, partial wave should hold
// the lightest tiles; else in index order, which keeps the tiles of one
// (b, h) together and their K/V shared in L2.  Launched with kOrderThreads
// threads per block: each thread takes kCostBins / kOrderThreads adjacent
// bins, and the bin offsets come from one block-wide scan.
constexpr int kOrderThreads = 1024;

__global__ void __launch_bounds__(kOrderThreads) tile_order_kernel(const int* __restrict__ cost,
                                                                   long long T, long long few_waves,
                                                                   int* __restrict__ order) {
  constexpr int kPer = kCostBins / kOrderThreads;  // bins per thread
  constexpr int kOrderWarps = kOrderThreads / 32;
  static_assert(kCostBins % kOrderThreads == 0, "bins split evenly over the threads");
  __shared__ int hist[kCostBins];
  __shared__ long long warp_total[kOrderWarps];
  __shared__ int warp_count[kOrderWarps], warp_top[kOrderWarps];
  __shared__ int sorted;
  const int* c = cost + blockIdx.x * T;
  int* o = order + blockIdx.x * T;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int b = tid; b < kCostBins; b += kOrderThreads) hist[b] = 0;
  __syncthreads();
  for (long long t = tid; t < T; t += kOrderThreads) atomicAdd(&hist[c[t]], 1);
  __syncthreads();
  // This thread's bins, heaviest first: kCostBins-1 - (tid*kPer + i).
  int cnt[kPer];
  int n = 0, top = 0;
  long long total = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int b = kCostBins - 1 - (tid * kPer + i);
    cnt[i] = hist[b];
    n += cnt[i];
    total += static_cast<long long>(b) * cnt[i];
    if (cnt[i] > 0) top = max(top, b);
  }
  int incl = n;  // inclusive scan of the counts in thread order (descending bins)
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += x;
  }
  long long wt = total;
  int wtop = top;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    wt += __shfl_xor_sync(0xffffffffu, wt, off);
    wtop = max(wtop, __shfl_xor_sync(0xffffffffu, wtop, off));
  }
  if (lane == 31) warp_count[warp] = incl;
  if (lane == 0) {
    warp_total[warp] = wt;
    warp_top[warp] = wtop;
  }
  __syncthreads();
  int run = incl - n;
  for (int w = 0; w < warp; ++w) run += warp_count[w];
  if (tid == 0) {
    long long all = 0;
    int heaviest = 0;
    for (int w = 0; w < kOrderWarps; ++w) {
      all += warp_total[w];
      heaviest = max(heaviest, warp_top[w]);
    }
    sorted = static_cast<long long>(heaviest) * T > 2 * all || T < few_waves;
  }
  __syncthreads();  // every thread has read its counts before the offsets overwrite them
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    hist[kCostBins - 1 - (tid * kPer + i)] = run;  // exclusive offset, heaviest bin first
    run += cnt[i];
  }
  __syncthreads();
  if (sorted) {
    for (long long t = tid; t < T; t += kOrderThreads)
      o[atomicAdd(&hist[c[t]], 1)] = static_cast<int>(t);
  } else {
    for (long long t = tid; t < T; t += kOrderThreads) o[t] = static_cast<int>(t);
  }
}

// Loads the R blocks blk[0..R) (block index, or -1 for a zero-filled pad)
// of a [B*H, N, D] tensor as one 128-row tile.
template <int BS, int D>
__device__ __forceinline__ void load_blocks(unsigned char* dst, const CUtensorMap* map,
                                            uint64_t* bar, const int* blk, int N, int bh) {
  using C = Cfg<BS, D>;
#pragma unroll
  for (int r = 0; r < C::R; ++r) {
    const int row0 = blk[r] >= 0 ? blk[r] * BS : N;  // past the end: the box reads zeros
#pragma unroll
    for (int ka = 0; ka < C::KATOMS; ++ka)
      tma_load_3d(dst + ka * C::ATOM + r * (BS * 128), map, bar, ka * 64, row0, bh);
  }
}

// S(+)= A . B^T with A, B 128-row K-major tiles in shared memory.
template <int D>
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false, false);
  const uint64_t ad0 = sdesc_sw128(a_smem, 16, 1024);
  const uint64_t bd0 = sdesc_sw128(b_smem, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
    umma_bf16_ss(d_tmem, ad0 + off, bd0 + off, kIdesc, kk > 0 ? 1u : 0u);
  }
}

// C(+)= A . B with A (128 x 128, bf16 packed two per column, the first 16 of
// every 32 columns) in TMEM and B a 128-row tile read MN-major (rows = K).
template <int D>
__device__ __forceinline__ void mma_ts(uint32_t c_tmem, uint32_t a_tmem, uint32_t b_smem,
                                       bool accumulate) {
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, D, false, true);
  const uint64_t bd0 = sdesc_sw128(b_smem, 128 * 128, 1024);
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk) {
    const uint32_t a_col = (kk >> 1) * 32 + (kk & 1) * 8;
    umma_bf16_ts(c_tmem, a_tmem + a_col, bd0 + ((kk * 16 * 128) >> 4), kIdesc,
                 (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Builds map[r] (the blocks listed by block kb0 + r of the CSR or CSC) and
// their union; blocks on the wrong side of the diagonal are dropped when
// causal (rows_side: the listed blocks are query blocks, keep i >= j).
__device__ void build_maps(Ctrl* ctl, const Args& a, int h, int kb0, int R, bool rows_side) {
  const int W = (a.M + 31) / 32;
  for (int w = threadIdx.x; w < W; w += blockDim.x) {
    ctl->uni[w] = 0u;
    for (int r = 0; r < R; ++r) ctl->map[r][w] = 0u;
  }
  __syncthreads();
  for (int r = 0; r < R; ++r) {
    const int own = kb0 + r;
    int e0 = a.ptr[static_cast<long long>(h) * a.M + own];
    int e1 = a.ptr[static_cast<long long>(h) * a.M + own + 1];
    if (e0 < 0 || e1 < e0) {
      if (threadIdx.x == 0) atomicOr(&g_bwd_status, BSA_STATUS_BAD_ROW_PTR);
      e0 = e1 = 0;
    }
    for (int e = e0 + static_cast<int>(threadIdx.x); e < e1; e += blockDim.x) {
      const int x = a.idx[e];
      if (x < 0 || x >= a.M) {
        atomicOr(&g_bwd_status, BSA_STATUS_BAD_COLUMN);
        continue;
      }
      if (a.causal && (rows_side ? x < own : x > own)) continue;
      atomicOr(&ctl->map[r][x >> 5], 1u << (x & 31));
      atomicOr(&ctl->uni[x >> 5], 1u << (x & 31));
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = 0;
    for (int w = 0; w < W; ++w) n += __popc(ctl->uni[w]);
    ctl->n_steps = (n + R - 1) / R;
  }
}

// Next up to R set bits of the union (ascending) into blk; -1 pads.
__device__ __forceinline__ void next_blocks(const Ctrl* ctl, int W, int& w, uint32_t& cur, int R,
                                            int* blk) {
  for (int r = 0; r < R; ++r) {
    while (cur == 0u && w + 1 < W) cur = ctl->uni[++w];
    if (cur == 0u) {
      blk[r] = -1;
    } else {
      blk[r] = w * 32 + __ffs(cur) - 1;
      cur &= cur - 1;
    }
  }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) { return pack_bf16x2(lo, hi); }

// Writes `groups` 32-column groups of this thread's accumulator row (fp32
// TMEM columns from `col`), times `mul`, as bf16 to out[row, ocol..].
__device__ __forceinline__ void store_groups(uint32_t tmem_lane, int col, int groups, float mul,
                                             __nv_bfloat16* out, long long row, int D, int ocol) {
  for (int g = 0; g < groups; ++g) {
    uint32_t r[32];
    tmem_ld32(tmem_lane + col + 32 * g, r);
    tmem_wait_ld();
    reg_fence32(r);
    uint4 v[4];
    uint32_t* w = reinterpret_cast<uint32_t*>(v);
#pragma unroll
    for (int c = 0; c < 16; ++c)
      w[c] = pack2(__uint_as_float(r[2 * c]) * mul, __uint_as_float(r[2 * c + 1]) * mul);
    uint4* dst = reinterpret_cast<uint4*>(out + row * D + ocol + 32 * g);
#pragma unroll
    for (int c = 0; c < 4; ++c) dst[c] = v[c];
  }
}

__device__ __forceinline__ void store_zero_cols(__nv_bfloat16* out, long long row, int D, int ocol,
                                                int n) {
  uint4* dst = reinterpret_cast<uint4*>(out + row * D + ocol);
  for (int c = 0; c < n / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
}

// Thread 0's view of the gathered-tile ring: two buffers, the k-th load of
// buffer b completes phase k of ld_bar[b].
struct Gather {
  int uw = 0;
  uint32_t ucur = 0;
  int issued[2] = {0, 0};
  int pending = 0;  // bit b: a load of buffer b not yet waited for
};

// ------------------------------------------------------------ dK, dV
// Step s uses buffer s & 1; the gather of step s + 1 is issued as soon as
// step s - 1's accumulating MMAs (the last readers of that buffer) are done,
// so it lands while step s computes.
template <int BS, int D>
__global__ void __launch_bounds__(kThreads, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tQ, const __grid_constant__ CUtensorMap tK,
                const __grid_constant__ CUtensorMap tV, const __grid_constant__ CUtensorMap tdO,
                const Args a) {
  using C = Cfg<BS, D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sK = smem;
  unsigned char* sV = smem + C::TILE;
  unsigned char* sQ = smem + 2 * C::TILE;   // two buffers
  unsigned char* sdO = smem + 4 * C::TILE;  // two buffers
  Ctrl* ctl = reinterpret_cast<Ctrl*>(smem + 6 * C::TILE);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;  // TMEM lane quadrant, column half
  const int tiles = a.N / 128;
  const int tile_id = a.order[blockIdx.x];
  const int bh = tile_id / tiles;
  const int kt = tile_id % tiles;
  const int h = bh % a.H;
  const int kb0 = kt * C::R;
  const int W = (a.M + 31) / 32;

  if (warp == 0) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&ctl->kv_bar, 1);
    mbar_init(&ctl->ld_bar[0], 1);
    mbar_init(&ctl->ld_bar[1], 1);
    mbar_init(&ctl->mma_bar, 1);
    mbar_init(&ctl->mma2_bar, 1);
    mbar_init(&ctl->final_bar, 1);
    fence_mbar_init();
    ctl->abort = 0;
  }
  build_maps(ctl, a, h, kb0, C::R, true);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const uint32_t tlane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const int steps = ctl->n_steps;

  Gather gt;
  gt.ucur = ctl->uni[0];
  auto gather = [&](int st) {  // thread 0: the tiles of step st into buffer st & 1
    const int b = st & 1;
    int blk[4];
    next_blocks(ctl, W, gt.uw, gt.ucur, C::R, blk);
    for (int r = 0; r < C::R; ++r) ctl->blk[b][r] = blk[r];
    mbar_arrive_expect_tx(&ctl->ld_bar[b], 2 * C::TILE);
    load_blocks<BS, D>(sQ + b * C::TILE, &tQ, &ctl->ld_bar[b], blk, a.N, bh);
    load_blocks<BS, D>(sdO + b * C::TILE, &tdO, &ctl->ld_bar[b], blk, a.N, bh);
    ++gt.issued[b];
    gt.pending |= 1 << b;
  };
  if (tid == 0 && steps > 0) {
    int own[4];
    for (int r = 0; r < C::R; ++r) own[r] = kb0 + r;
    mbar_arrive_expect_tx(&ctl->kv_bar, 2 * C::TILE);
    load_blocks<BS, D>(sK, &tK, &ctl->kv_bar, own, a.N, bh);
    load_blocks<BS, D>(sV, &tV, &ctl->kv_bar, own, a.N, bh);
    gather(0);
  }

  const int k = quad * 32 + lane;           // key row of the tile
  const int kb = k / BS;                    // its block within the tile
  const int ktok = kt * 128 + k;
  int done = 0;                             // steps whose accumulating MMAs were issued
  for (int s = 0; s < steps; ++s) {
    const int b = s & 1;
    if (tid == 0) {
      if (s > 0 && !wait_bounded(&ctl->mma2_bar, (s - 1) & 1, &ctl->abort)) {
        // nothing more is issued; the teardown drains
      } else if (s + 1 < steps) {
        gather(s + 1);
      }
    }
    __syncthreads();
    if (ctl->abort) break;
    if (tid < 128) {
      const int r = tid / BS;
      const int qb = ctl->blk[b][r];
      if (qb >= 0) {
        const long long q = static_cast<long long>(bh) * a.N + qb * BS + tid % BS;
        ctl->lse2[tid] = a.LSE[q] * kLog2e;
        ctl->dd[tid] = a.Dq[q];
      } else {
        ctl->lse2[tid] = 0.f;
        ctl->dd[tid] = 0.f;
      }
    }
    if (tid == 0) {
      bool ok = !(s == 0 && !wait_bounded(&ctl->kv_bar, 0, &ctl->abort));
      ok = ok && wait_bounded(&ctl->ld_bar[b], (s >> 1) & 1, &ctl->abort);
      if (ok) {
        gt.pending &= ~(1 << b);
        tc_fence_after();
        mma_ss<D>(tmem + C::TMEM_A, smem_u32(sK), smem_u32(sQ + b * C::TILE));   // S^T = K Q^T
        mma_ss<D>(tmem + C::TMEM_B, smem_u32(sV), smem_u32(sdO + b * C::TILE));  // dP^T = V dO^T
        umma_commit(&ctl->mma_bar);
      }
    }
    wait_bounded(&ctl->mma_bar, s & 1, &ctl->abort);
    __syncthreads();
    if (ctl->abort) break;
    tc_fence_after();

    // this key row against 64 of the step's 128 queries, 32 at a time
    bool member[4];
    int qb0[4];
#pragma unroll
    for (int r = 0; r < C::R; ++r) {
      qb0[r] = ctl->blk[b][r];
      member[r] = qb0[r] >= 0 && ((ctl->map[kb][qb0[r] >> 5] >> (qb0[r] & 31)) & 1u);
    }
#pragma unroll 1
    for (int gg = 0; gg < 2; ++gg) {
      const int g = half * 2 + gg;
      // A 32-column group lies inside one block of the step, and a warp's 32
      // rows inside one block of the tile (BS >= 32): whether the pair is in
      // the pattern is uniform over the warp.  Groups outside it only write
      // zeros.
      const int rg = (32 * g) / BS;
      const bool mem_g = member[rg];
      uint32_t pp[16], dp[16];
      if (mem_g) {
        uint32_t sr[32], dr[32];
        tmem_ld32(tlane + C::TMEM_A + 32 * g, sr);
        tmem_ld32(tlane + C::TMEM_B + 32 * g, dr);
        tmem_wait_ld();
        reg_fence32(sr);
        reg_fence32(dr);
        const int qtok0 = qb0[rg] * BS + (32 * g) % BS;
        const float4* l4 = reinterpret_cast<const float4*>(ctl->lse2 + 32 * g);
        const float4* d4 = reinterpret_cast<const float4*>(ctl->dd + 32 * g);
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 lq = l4[c / 4], dq = d4[c / 4];
          const float lv[4] = {lq.x, lq.y, lq.z, lq.w}, dvv[4] = {dq.x, dq.y, dq.z, dq.w};
          float pv[4], dv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const bool allowed = !a.causal || qtok0 + c + e >= ktok;
            const float p = allowed ? ex2_approx(fmaf(__uint_as_float(sr[c + e]), a.scale_log2,
                                                      -lv[e]))
                                    : 0.f;
            pv[e] = p;
            dv[e] = p * (__uint_as_float(dr[c + e]) - dvv[e]);
          }
          pp[c / 2] = pack2(pv[0], pv[1]);
          pp[c / 2 + 1] = pack2(pv[2], pv[3]);
          dp[c / 2] = pack2(dv[0], dv[1]);
          dp[c / 2 + 1] = pack2(dv[2], dv[3]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) pp[c] = dp[c] = 0u;
      }
      tmem_st16(tlane + C::TMEM_A + 32 * g, pp);   // P^T over consumed S^T columns
      tmem_st16(tlane + C::TMEM_B + 32 * g, dp);   // dS^T over consumed dP^T columns
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      mma_ts<D>(tmem + C::TMEM_C, tmem + C::TMEM_A, smem_u32(sdO + b * C::TILE), s > 0);  // dV
      mma_ts<D>(tmem + C::TMEM_D, tmem + C::TMEM_B, smem_u32(sQ + b * C::TILE), s > 0);   // dK
      umma_commit(&ctl->mma2_bar);
    }
    done = s + 1;
  }

  // teardown: every copy and MMA issued must complete before TMEM is freed
  // and before the CTA's shared memory goes away
  if (tid == 0) {
    umma_commit(&ctl->final_bar);  // arrives once every MMA issued so far has completed
    wait_drain(&ctl->final_bar, 0);
    for (int b = 0; b < 2; ++b)
      if (gt.pending & (1 << b)) wait_drain(&ctl->ld_bar[b], (gt.issued[b] - 1) & 1);
    if (steps > 0) wait_drain(&ctl->kv_bar, 0);
  }
  __syncthreads();
  tc_fence_after();
  const long long row = static_cast<long long>(bh) * a.N + ktok;
  if (!ctl->abort) {
    const int ocol = half * (D / 2);
    if (done == 0) {
      store_zero_cols(a.out0, row, D, ocol, D / 2);
      store_zero_cols(a.out1, row, D, ocol, D / 2);
    } else {
      store_groups(tlane, C::TMEM_C + ocol, D / 64, 1.f, a.out0, row, D, ocol);
      store_groups(tlane, C::TMEM_D + ocol, D / 64, a.scale, a.out1, row, D, ocol);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------- dQ
template <int BS, int D>
__global__ void __launch_bounds__(kThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tQ, const __grid_constant__ CUtensorMap tK,
              const __grid_constant__ CUtensorMap tV, const __grid_constant__ CUtensorMap tdO,
              const Args a) {
  using C = Cfg<BS, D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = smem;
  unsigned char* sdO = smem + C::TILE;
  unsigned char* sK = smem + 2 * C::TILE;  // two buffers
  unsigned char* sV = smem + 4 * C::TILE;  // two buffers
  Ctrl* ctl = reinterpret_cast<Ctrl*>(smem + 6 * C::TILE);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int tiles = a.N / 128;
  const int tile_id = a.order[blockIdx.x];
  const int bh = tile_id / tiles;
  const int qt = tile_id % tiles;
  const int h = bh % a.H;
  const int rb0 = qt * C::R;
  const int W = (a.M + 31) / 32;

  if (warp == 0) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&ctl->kv_bar, 1);
    mbar_init(&ctl->ld_bar[0], 1);
    mbar_init(&ctl->ld_bar[1], 1);
    mbar_init(&ctl->mma_bar, 1);
    mbar_init(&ctl->mma2_bar, 1);
    mbar_init(&ctl->final_bar, 1);
    fence_mbar_init();
    ctl->abort = 0;
  }
  build_maps(ctl, a, h, rb0, C::R, false);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const uint32_t tlane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const int steps = ctl->n_steps;

  const int q = quad * 32 + lane;    // query row of the tile
  const int rb = q / BS;             // its block row within the tile
  const int qtok = qt * 128 + q;
  const long long qrow = static_cast<long long>(bh) * a.N + qtok;
  const float lse2 = a.LSE[qrow] * kLog2e;
  const float dq_d = a.Dq[qrow];

  Gather gt;
  gt.ucur = ctl->uni[0];
  auto gather = [&](int st) {
    const int b = st & 1;
    int blk[4];
    next_blocks(ctl, W, gt.uw, gt.ucur, C::R, blk);
    for (int r = 0; r < C::R; ++r) ctl->blk[b][r] = blk[r];
    mbar_arrive_expect_tx(&ctl->ld_bar[b], 2 * C::TILE);
    load_blocks<BS, D>(sK + b * C::TILE, &tK, &ctl->ld_bar[b], blk, a.N, bh);
    load_blocks<BS, D>(sV + b * C::TILE, &tV, &ctl->ld_bar[b], blk, a.N, bh);
    ++gt.issued[b];
    gt.pending |= 1 << b;
  };
  if (tid == 0 && steps > 0) {
    int own[4];
    for (int r = 0; r < C::R; ++r) own[r] = rb0 + r;
    mbar_arrive_expect_tx(&ctl->kv_bar, 2 * C::TILE);
    load_blocks<BS, D>(sQ, &tQ, &ctl->kv_bar, own, a.N, bh);
    load_blocks<BS, D>(sdO, &tdO, &ctl->kv_bar, own, a.N, bh);
    gather(0);
  }
  int done = 0;
  for (int s = 0; s < steps; ++s) {
    const int b = s & 1;
    if (tid == 0) {
      if (s > 0 && !wait_bounded(&ctl->mma2_bar, (s - 1) & 1, &ctl->abort)) {
      } else if (s + 1 < steps) {
        gather(s + 1);
      }
    }
    __syncthreads();
    if (ctl->abort) break;
    if (tid == 0) {
      bool ok = !(s == 0 && !wait_bounded(&ctl->kv_bar, 0, &ctl->abort));
      ok = ok && wait_bounded(&ctl->ld_bar[b], (s >> 1) & 1, &ctl->abort);
      if (ok) {
        gt.pending &= ~(1 << b);
        tc_fence_after();
        mma_ss<D>(tmem + C::TMEM_A, smem_u32(sQ), smem_u32(sK + b * C::TILE));   // S = Q K^T
        mma_ss<D>(tmem + C::TMEM_B, smem_u32(sdO), smem_u32(sV + b * C::TILE));  // dP = dO V^T
        umma_commit(&ctl->mma_bar);
      }
    }
    wait_bounded(&ctl->mma_bar, s & 1, &ctl->abort);
    __syncthreads();
    if (ctl->abort) break;
    tc_fence_after();

    bool member[4];
    int kb0[4];
#pragma unroll
    for (int r = 0; r < C::R; ++r) {
      kb0[r] = ctl->blk[b][r];
      member[r] = kb0[r] >= 0 && ((ctl->map[rb][kb0[r] >> 5] >> (kb0[r] & 31)) & 1u);
    }
#pragma unroll 1
    for (int gg = 0; gg < 2; ++gg) {
      const int g = half * 2 + gg;
      // the pair (block row, key block of the group) is uniform over the warp
      const int rg = (32 * g) / BS;
      const bool mem_g = member[rg];
      uint32_t dp[16];
      if (mem_g) {
        uint32_t sr[32], dr[32];
        tmem_ld32(tlane + C::TMEM_A + 32 * g, sr);
        tmem_ld32(tlane + C::TMEM_B + 32 * g, dr);
        tmem_wait_ld();
        reg_fence32(sr);
        reg_fence32(dr);
        const int ktok0 = kb0[rg] * BS + (32 * g) % BS;
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float dv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool allowed = !a.causal || ktok0 + c + e <= qtok;
            const float p = allowed ? ex2_approx(fmaf(__uint_as_float(sr[c + e]), a.scale_log2,
                                                      -lse2))
                                    : 0.f;
            dv[e] = p * (__uint_as_float(dr[c + e]) - dq_d);
          }
          dp[c / 2] = pack2(dv[0], dv[1]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) dp[c] = 0u;
      }
      tmem_st16(tlane + C::TMEM_A + 32 * g, dp);   // dS over consumed S columns
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      mma_ts<D>(tmem + C::TMEM_C, tmem + C::TMEM_A, smem_u32(sK + b * C::TILE), s > 0);  // dQ += dS K
      umma_commit(&ctl->mma2_bar);
    }
    done = s + 1;
  }

  if (tid == 0) {
    umma_commit(&ctl->final_bar);
    wait_drain(&ctl->final_bar, 0);
    for (int b = 0; b < 2; ++b)
      if (gt.pending & (1 << b)) wait_drain(&ctl->ld_bar[b], (gt.issued[b] - 1) & 1);
    if (steps > 0) wait_drain(&ctl->kv_bar, 0);
  }
  __syncthreads();
  tc_fence_after();
  if (!ctl->abort) {
    const int ocol = half * (D / 2);
    if (done == 0)
      store_zero_cols(a.out0, qrow, D, ocol, D / 2);
    else
      store_groups(tlane, C::TMEM_C + ocol, D / 64, a.scale, a.out0, qrow, D, ocol);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B*H, N, d] bf16 as a 3-D tensor; box = 64 columns x `rows` rows x 1.
bool make_map(CUtensorMap* m, const void* base, long long BH, int N, int d, int rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BS, int D>
int launch(const void* Q, const void* K, const void* V, const void* dO, Args a, long long BH,
           const int32_t* row_ptr, const int32_t* col_idx, const int32_t* col_ptr,
           const int32_t* row_idx, void* dQ, void* dK, void* dV, int* cost, int* order,
           cudaStream_t s) {
  using C = Cfg<BS, D>;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map(&tq, Q, BH, a.N, D, BS) || !make_map(&tk, K, BH, a.N, D, BS) ||
      !make_map(&tv, V, BH, a.N, D, BS) || !make_map(&tdo, dO, BH, a.N, D, BS))
    return BSA_ERR_CUDA;
  // At least ~120 KB, so that one CTA (and its 512 TMEM columns) owns each SM.
  int smem = 6 * C::TILE + static_cast<int>(sizeof(Ctrl)) + 1024;
  if (smem < 120 * 1024) smem = 120 * 1024;
  if (cudaFuncSetAttribute(dkdv_kernel<BS, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess ||
      cudaFuncSetAttribute(dq_kernel<BS, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess)
    return BSA_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(BH * (a.N / 128));
  const long long T = static_cast<long long>(grid);
  // order[0..T): key tiles by their column lists; order[T..2T): query tiles by their rows
  tile_cost_kernel<<<static_cast<unsigned>((T + 255) / 256), 256, 0, s>>>(
      col_ptr, row_ptr, a.H, a.M, C::R, a.N / 128, T, cost);
  if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  tile_order_kernel<<<2, kOrderThreads, 0, s>>>(cost, T, 8LL * sms, order);
  if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  Args kv = a;
  kv.ptr = col_ptr;
  kv.idx = row_idx;
  kv.out0 = static_cast<__nv_bfloat16*>(dV);
  kv.out1 = static_cast<__nv_bfloat16*>(dK);
  kv.order = order;
  dkdv_kernel<BS, D><<<grid, kThreads, smem, s>>>(tq, tk, tv, tdo, kv);
  if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  Args qa = a;
  qa.ptr = row_ptr;
  qa.idx = col_idx;
  qa.out0 = static_cast<__nv_bfloat16*>(dQ);
  qa.out1 = nullptr;
  qa.order = order + T;
  dq_kernel<BS, D><<<grid, kThreads, smem, s>>>(tq, tk, tv, tdo, qa);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace bwd
}  // namespace bsa

// D (fp32 per query row), then the tile costs and the two tile orders (int
// per 128-row tile, twice each).
extern "C" size_t bsa_backward_workspace_bytes(int B, int H, int N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  const size_t rows = static_cast<size_t>(B) * static_cast<size_t>(H) * static_cast<size_t>(N);
  const size_t tiles = static_cast<size_t>(B) * static_cast<size_t>(H) * ((N + 127) / 128);
  return rows * sizeof(float) + 4 * tiles * sizeof(int);
}

extern "C" int bsa_backward(const void* Q, const void* K, const void* V, const void* O,
                            const void* dO, const float* LSE, const int32_t* row_ptr,
                            const int32_t* col_idx, const int32_t* col_ptr,
                            const int32_t* row_idx, int B, int H, int N, int d, int block_size,
                            float scale, int causal, void* dQ, void* dK, void* dV,
                            void* workspace, size_t workspace_bytes, void* stream) {
  using namespace bsa::bwd;
  if (!Q || !K || !V || !O || !dO || !LSE || !row_ptr || !col_idx || !col_ptr || !row_idx ||
      !dQ || !dK || !dV || !workspace)
    return BSA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || d < 1 || block_size < 1) return BSA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return BSA_ERR_INVALID_ARG;
  if (N % block_size != 0 || !std::isfinite(scale)) return BSA_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, O, dO, dQ, dK, dV};
  for (const void* p : ptrs)
    if (!aligned16(p)) return BSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(LSE) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
    return BSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BSA_ERR_UNSUPPORTED;
  if (block_size != 32 && block_size != 64 && block_size != 128) return BSA_ERR_UNSUPPORTED;
  if (N % 128 != 0) return BSA_ERR_UNSUPPORTED;
  const int M = N / block_size;
  if (M > kMaxM) return BSA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  if (BH * (N / 128) > 0x7fffffffLL || BH * N > (1LL << 40)) return BSA_ERR_UNSUPPORTED;
  if (workspace_bytes < bsa_backward_workspace_bytes(B, H, N)) return BSA_ERR_BUFFER_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* Dq = static_cast<float*>(workspace);
  int* cost = reinterpret_cast<int*>(Dq + BH * N);
  int* order = cost + 2 * BH * (N / 128);
  const long long rows = BH * N;
  const int threads = 256;
  long long blocks = (rows * (d / 8) + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  dot_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO), Dq, rows, d);
  if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  Args a;
  a.LSE = LSE;
  a.Dq = Dq;
  a.H = H;
  a.N = N;
  a.M = M;
  a.scale = scale;
  a.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  a.causal = causal;
  const int key = block_size * 1000 + d;
  switch (key) {
    case 32064: return launch<32, 64>(Q, K, V, dO, a, BH, row_ptr, col_idx, col_ptr, row_idx, dQ, dK, dV, cost, order, s);
    case 32128: return launch<32, 128>(Q, K, V, dO, a, BH, row_ptr, col_idx, col_ptr, row_idx, dQ, dK, dV, cost, order, s);
    case 64064: return launch<64, 64>(Q, K, V, dO, a, BH, row_ptr, col_idx, col_ptr, row_idx, dQ, dK, dV, cost, order, s);
    case 64128: return launch<64, 128>(Q, K, V, dO, a, BH, row_ptr, col_idx, col_ptr, row_idx, dQ, dK, dV, cost, order, s);
    case 128064: return launch<128, 64>(Q, K, V, dO, a, BH, row_ptr, col_idx, col_ptr, row_idx, dQ, dK, dV, cost, order, s);
    case 128128: return launch<128, 128>(Q, K, V, dO, a, BH, row_ptr, col_idx, col_ptr, row_idx, dQ, dK, dV, cost, order, s);
    default: return BSA_ERR_UNSUPPORTED;
  }
}

extern "C" int bsa_backward_status(uint32_t* status, int clear) {
  if (!status) return BSA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return BSA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, bsa::bwd::g_bwd_status, sizeof(v)) != cudaSuccess)
    return BSA_ERR_CUDA;
  if (clear) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(bsa::bwd::g_bwd_status, &z, sizeof(z)) != cudaSuccess)
      return BSA_ERR_CUDA;
  }
  *status = v;
  return BSA_OK;
}
