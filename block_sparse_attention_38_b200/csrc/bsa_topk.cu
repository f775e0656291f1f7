// bsa_topk.cu -- content-based top-k block selection on the device.
//
// The SparseFlashAttention article ("pattern generation", third kind) picks
// the Top-K positions by the similarity of Q and K; here, at block level, row
// i keeps its diagonal block and the top_k blocks j (j != i, j <= i when
// causal) of highest s[i, j] = Qm[i] . Km[j], Qm and Km the block means of Q
// and K.  The selection is an integer decision, so the arithmetic is pinned
// to fp64 in a fixed order with every operation rounded on its own
// (__dadd_rn / __dmul_rn: no fused multiply-add): tokens added in ascending
// order, then products over c in ascending order.
//
//   means_kernel   one CTA per (bh, block), one thread per column c; the K
//                  means are stored transposed, [bh][c][block], so that the
//                  threads of the selection (one per candidate block) read
//                  consecutive addresses for each c
//   select_warp_kernel  (M <= 1024) one warp per (bh, block row): the
//                  candidates' scores, a bitonic sort and the selection, all
//                  in registers (see below)
//   select_kernel  (larger M) one CTA per (bh, block row): scores of the M
//                  candidate blocks into shared memory, a bitonic sort on
//                  (score descending, column ascending), then the chosen
//                  columns written in ascending order at the row's fixed CSR
//                  offset
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "bsa.h"

namespace bsa {
namespace topk {

constexpr int kMaxM = 4096;
constexpr int kMaxD = 256;
constexpr int kSelectThreads = 256;

__host__ __device__ inline int64_t row_length(int64_t i, int64_t M, int64_t top_k, int causal) {
  const int64_t others = causal ? i : M - 1;
  return 1 + (top_k < others ? top_k : others);
}

// Stored blocks of rows 0..i-1 of one (bh).
__host__ __device__ inline int64_t row_offset(int64_t i, int64_t M, int64_t top_k, int causal) {
  if (!causal) return i * (1 + (top_k < M - 1 ? top_k : M - 1));
  // sum over i' < i of 1 + min(top_k, i')
  const int64_t m = i < top_k ? i : top_k;
  const int64_t tail = i > top_k ? (i - top_k) * top_k : 0;
  return i + m * (m - 1) / 2 + tail;
}

// qm: [BH, M, d];  kmT: [BH, d, M].
__global__ void means_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                             int M, int d, int bs, double* __restrict__ qm,
                             double* __restrict__ kmT) {
  const long long blk = blockIdx.x;  // bh * M + i: tokens blk*bs .. blk*bs + bs - 1
  const long long bh = blk / M;
  const int i = static_cast<int>(blk - bh * M);
  const int c = threadIdx.x;
  if (c >= d) return;
  const long long base = blk * bs * d + c;
  double sq = 0.0, sk = 0.0;
  for (int t = 0; t < bs; ++t) {
    sq = __dadd_rn(sq, static_cast<double>(__bfloat162float(Q[base + static_cast<long long>(t) * d])));
    sk = __dadd_rn(sk, static_cast<double>(__bfloat162float(K[base + static_cast<long long>(t) * d])));
  }
  const double inv = 1.0 / bs;  // exact: bs is a power of two in practice, and the oracle divides
  qm[blk * d + c] = bs == (bs & -bs) ? __dmul_rn(sq, inv) : __ddiv_rn(sq, static_cast<double>(bs));
  kmT[(bh * d + c) * M + i] = bs == (bs & -bs) ? __dmul_rn(sk, inv) : __ddiv_rn(sk, static_cast<double>(bs));
}

// a before b: higher score, then smaller column.
__device__ inline bool before(double sa, int ja, double sb, int jb) {
  return sa > sb || (sa == sb && ja < jb);
}

__global__ void __launch_bounds__(kSelectThreads)
    select_kernel(const double* __restrict__ qm, const double* __restrict__ kmT, int M, int Mp,
                  int d, int top_k, int causal, int32_t* __restrict__ row_ptr,
                  int32_t* __restrict__ col_idx, long long num_rows) {
  extern __shared__ unsigned char smem_raw[];
  double* score = reinterpret_cast<double*>(smem_raw);          // [Mp]
  double* qrow = score + Mp;                                   // [d]
  int* idx = reinterpret_cast<int*>(qrow + kMaxD);             // [Mp]
  unsigned char* chosen = reinterpret_cast<unsigned char*>(idx + Mp);  // [Mp]
  __shared__ int warp_sum[kSelectThreads / 32];

  const long long r = blockIdx.x;  // bh * M + i
  const long long bh = r / M;
  const int i = static_cast<int>(r - bh * M);
  const int tid = threadIdx.x;
  for (int c = tid; c < d; c += kSelectThreads) qrow[c] = qm[r * d + c];
  __syncthreads();

  const double* kbase = kmT + bh * static_cast<long long>(M) * d;
  for (int j = tid; j < Mp; j += kSelectThreads) {
    double s = -INFINITY;  // not a candidate: sorts after every finite score
    if (j < M && j != i && (!causal || j <= i)) {
      s = 0.0;
      const double* kc = kbase + j;  // Km[j, c] at kc[c * M]
      for (int c = 0; c < d; ++c) s = __dadd_rn(s, __dmul_rn(qrow[c], kc[static_cast<long long>(c) * M]));
    }
    score[j] = s;
    idx[j] = j;
    chosen[j] = 0;
  }
  __syncthreads();

  // Bitonic sort of (score, column) over Mp (a power of two) entries.
  for (int size = 2; size <= Mp; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int p = tid; p < Mp / 2; p += kSelectThreads) {
        const int lo = 2 * p - (p & (stride - 1));  // first element of the pair
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;           // this run sorts in "before" order
        const bool swap = up ? before(score[hi], idx[hi], score[lo], idx[lo])
                             : before(score[lo], idx[lo], score[hi], idx[hi]);
        if (swap) {
          const double ts = score[lo];
          score[lo] = score[hi];
          score[hi] = ts;
          const int ti = idx[lo];
          idx[lo] = idx[hi];
          idx[hi] = ti;
        }
      }
      __syncthreads();
    }
  }

  const int keep = static_cast<int>(row_length(i, M, top_k, causal)) - 1;  // chosen besides i
  for (int p = tid; p < keep; p += kSelectThreads) chosen[idx[p]] = 1;
  if (tid == 0) chosen[i] = 1;
  __syncthreads();

  // Chosen columns in ascending order: each thread owns a contiguous range.
  const int per = (M + kSelectThreads - 1) / kSelectThreads;
  const int j0 = tid * per, j1 = min(M, j0 + per);
  int cnt = 0;
  for (int j = j0; j < j1; ++j) cnt += chosen[j];
  const int lane = tid & 31, warp = tid >> 5;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_sum[w];
  const long long row_start = bh * row_offset(M, M, top_k, causal) + row_offset(i, M, top_k, causal);
  int pos = base + incl - cnt;
  for (int j = j0; j < j1; ++j)
    if (chosen[j]) col_idx[row_start + pos++] = j;
  if (tid == 0) {
    row_ptr[r] = static_cast<int32_t>(row_start);
    if (r == num_rows - 1)
      row_ptr[num_rows] = static_cast<int32_t>(row_start + row_length(i, M, top_k, causal));
  }
}

// One warp per (bh, block row) for M <= 1024: lane l takes the candidates
// j = l + 32e (e < E, E = Mp / 32), scores them with the same fixed-order fp64
// chain as select_kernel (E independent chains per lane), sorts the Mp
// (score, column) pairs with a bitonic network held in registers (pairs 32
// or more apart swap inside a lane, closer ones between lanes by shuffle),
// marks the first `keep` columns and the diagonal in a per-warp bitmap, and
// writes the marked columns in ascending order.
constexpr int kWarpRowsPerCta = 8;

template <int E>
__global__ void __launch_bounds__(32 * kWarpRowsPerCta)
    select_warp_kernel(const double* __restrict__ qm, const double* __restrict__ kmT, int M, int d,
                       int top_k, int causal, int32_t* __restrict__ row_ptr,
                       int32_t* __restrict__ col_idx, long long num_rows) {
  __shared__ uint32_t marks[kWarpRowsPerCta][32];
  const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
  const long long r = static_cast<long long>(blockIdx.x) * kWarpRowsPerCta + wl;  // bh * M + i
  if (r >= num_rows) return;
  const long long bh = r / M;
  const int i = static_cast<int>(r - bh * M);
  const double* qrow = qm + r * d;
  const double* kbase = kmT + bh * static_cast<long long>(M) * d;

  double sc[E];
  int col[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    col[e] = lane + 32 * e;
    sc[e] = 0.0;
  }
  // U columns c per round: all their loads are issued before the first of
  // their products, so one round costs one memory latency; the sums still
  // run over c in ascending order.
  constexpr int U = E >= 32 ? 1 : 32 / E;  // 32 loads in flight per lane and round
  for (int c0 = 0; c0 < d; c0 += U) {
    double qv[U], kv[U][E];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u;
      qv[u] = c < d ? __ldg(qrow + c) : 0.0;
      const double* kc = kbase + static_cast<long long>(c) * M;
#pragma unroll
      for (int e = 0; e < E; ++e) kv[u][e] = (c < d && col[e] < M) ? __ldg(kc + col[e]) : 0.0;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (c0 + u >= d) break;
#pragma unroll
      for (int e = 0; e < E; ++e)
        if (col[e] < M) sc[e] = __dadd_rn(sc[e], __dmul_rn(qv[u], kv[u][e]));
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int j = col[e];
    if (j >= M || j == i || (causal && j > i)) sc[e] = -INFINITY;  // not a candidate: sorts last
  }

  // Bitonic sort into "before" order (higher score, then smaller column).
  constexpr int Mp = 32 * E;
#pragma unroll
  for (int size = 2; size <= Mp; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= 32) {  // partners in the same lane: registers e and e ^ (stride / 32)
        const int es = stride / 32;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          if (e & es) continue;
          const int pos = lane + 32 * e;                 // the lower element of the pair
          const bool up = (pos & size) == 0;
          const int f = e | es;
          const bool swap = up ? before(sc[f], col[f], sc[e], col[e])
                               : before(sc[e], col[e], sc[f], col[f]);
          if (swap) {
            const double ts = sc[e]; sc[e] = sc[f]; sc[f] = ts;
            const int tc = col[e]; col[e] = col[f]; col[f] = tc;
          }
        }
      } else {  // partners in lanes lane ^ stride, same register
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const double os = __shfl_xor_sync(0xffffffffu, sc[e], stride);
          const int oc = __shfl_xor_sync(0xffffffffu, col[e], stride);
          const int pos = lane + 32 * e;
          const bool lower = (lane & stride) == 0;
          const bool up = (pos & size) == 0;
          // the lower element keeps the one that comes first in its run's order
          const bool other_first = before(os, oc, sc[e], col[e]);
          const bool take = (lower == up) ? other_first : !other_first;
          if (take) {
            sc[e] = os;
            col[e] = oc;
          }
        }
      }
    }
  }

  const int keep = static_cast<int>(row_length(i, M, top_k, causal)) - 1;  // chosen besides i
  marks[wl][lane] = 0u;
  __syncwarp();
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (lane + 32 * e < keep) atomicOr(&marks[wl][col[e] >> 5], 1u << (col[e] & 31));
  if (lane == 0) atomicOr(&marks[wl][i >> 5], 1u << (i & 31));
  __syncwarp();
  // Word `lane` holds columns 32 lane .. 32 lane + 31: ascending order by a warp scan.
  uint32_t word = marks[wl][lane];
  const int cnt = __popc(word);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const long long row_start = bh * row_offset(M, M, top_k, causal) + row_offset(i, M, top_k, causal);
  int pos = incl - cnt;
  while (word) {
    const int b = __ffs(word) - 1;
    word &= word - 1;
    col_idx[row_start + pos++] = lane * 32 + b;
  }
  if (lane == 0) {
    row_ptr[r] = static_cast<int32_t>(row_start);
    if (r == num_rows - 1)
      row_ptr[num_rows] = static_cast<int32_t>(row_start + row_length(i, M, top_k, causal));
  }
}

template <int E>
int launch_select_warp(const double* qm, const double* kmT, int M, int d, int top_k, int causal,
                       int32_t* row_ptr, int32_t* col_idx, long long rows, cudaStream_t s) {
  const long long grid = (rows + kWarpRowsPerCta - 1) / kWarpRowsPerCta;
  select_warp_kernel<E><<<static_cast<unsigned>(grid), 32 * kWarpRowsPerCta, 0, s>>>(
      qm, kmT, M, d, top_k, causal, row_ptr, col_idx, rows);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

}  // namespace topk
}  // namespace bsa

extern "C" int64_t bsa_topk_nnz(int BH, int M, int top_k, int causal) {
  if (BH < 1 || M < 1 || top_k < 0 || (causal != 0 && causal != 1)) return -1;
  return static_cast<int64_t>(BH) * bsa::topk::row_offset(M, M, top_k, causal);
}

extern "C" size_t bsa_topk_workspace_bytes(int BH, int N, int d, int block_size) {
  if (BH < 1 || N < 1 || d < 1 || block_size < 1 || N % block_size != 0) return 0;
  return 2ull * static_cast<size_t>(BH) * static_cast<size_t>(N / block_size) *
         static_cast<size_t>(d) * sizeof(double);
}

extern "C" int bsa_topk_pattern(const void* Q, const void* K, int BH, int N, int d,
                                int block_size, int top_k, int causal, int32_t* row_ptr,
                                int32_t* col_idx, void* workspace, size_t workspace_bytes,
                                void* stream) {
  using namespace bsa::topk;
  if (!Q || !K || !row_ptr || !col_idx || !workspace) return BSA_ERR_INVALID_ARG;
  if (BH < 1 || N < 1 || d < 1 || block_size < 1 || top_k < 0) return BSA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return BSA_ERR_INVALID_ARG;
  if (N % block_size != 0) return BSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 7u) != 0) return BSA_ERR_INVALID_ARG;
  const int M = N / block_size;
  if (d > kMaxD || M > kMaxM) return BSA_ERR_UNSUPPORTED;
  const int64_t nnz = bsa_topk_nnz(BH, M, top_k, causal);
  if (static_cast<int64_t>(BH) * M + 1 > INT32_MAX || nnz > INT32_MAX) return BSA_ERR_UNSUPPORTED;
  if (workspace_bytes < bsa_topk_workspace_bytes(BH, N, d, block_size)) return BSA_ERR_BUFFER_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* qm = static_cast<double*>(workspace);
  double* kmT = qm + static_cast<size_t>(BH) * M * d;
  const long long blocks = static_cast<long long>(BH) * M;
  means_kernel<<<static_cast<unsigned>(blocks), d, 0, s>>>(
      static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K), M, d, block_size,
      qm, kmT);
  if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  int Mp = 1;
  while (Mp < M) Mp <<= 1;
  if (Mp < 2) Mp = 2;
  if (Mp <= 1024) {  // one warp per row, everything in registers
    const int E = Mp <= 32 ? 1 : Mp / 32;
    switch (E) {
      case 1: return launch_select_warp<1>(qm, kmT, M, d, top_k, causal, row_ptr, col_idx, blocks, s);
      case 2: return launch_select_warp<2>(qm, kmT, M, d, top_k, causal, row_ptr, col_idx, blocks, s);
      case 4: return launch_select_warp<4>(qm, kmT, M, d, top_k, causal, row_ptr, col_idx, blocks, s);
      case 8: return launch_select_warp<8>(qm, kmT, M, d, top_k, causal, row_ptr, col_idx, blocks, s);
      case 16: return launch_select_warp<16>(qm, kmT, M, d, top_k, causal, row_ptr, col_idx, blocks, s);
      default: return launch_select_warp<32>(qm, kmT, M, d, top_k, causal, row_ptr, col_idx, blocks, s);
    }
  }
  const size_t smem = static_cast<size_t>(Mp) * sizeof(double) + kMaxD * sizeof(double) +
                      static_cast<size_t>(Mp) * sizeof(int) + static_cast<size_t>(Mp);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return BSA_ERR_CUDA;
  select_kernel<<<static_cast<unsigned>(blocks), kSelectThreads, smem, s>>>(
      qm, kmT, M, Mp, d, top_k, causal, row_ptr, col_idx, blocks);
  if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  return BSA_OK;
}

// ---------------------------------------------------------------------------
// bsa_topk_pattern_static: the same selection with its fp64 workspace in a
// fixed scratch area of this library instead of caller memory.  Every device
// gets its own copy of the array when the library's module loads there; its
// address is looked up once per device, on the first call, and kept for the
// life of the process (a device reset leaves it stale).  No element of the
// scratch needs to start at zero: the means kernel writes every element the
// selection then reads, within the same call.  Two calls that overlap in time
// on one device share the area and race.
namespace bsa {
namespace topk {

constexpr size_t kStaticScratchBytes = BSA_TOPK_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) double g_static_scratch[kStaticScratchBytes / sizeof(double)];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_static_addr[kMaxDevices];
std::mutex g_static_mu;

// Address of this device's scratch, or nullptr if the lookup failed.
void* static_scratch(int dev) {
  void* p = g_static_addr[dev].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lock(g_static_mu);
  p = g_static_addr[dev].load(std::memory_order_relaxed);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
    g_static_addr[dev].store(p, std::memory_order_release);
  }
  return p;
}

}  // namespace topk
}  // namespace bsa

extern "C" int bsa_topk_pattern_static(const void* Q, const void* K, int BH, int N, int d,
                                       int block_size, int top_k, int causal, int32_t* row_ptr,
                                       int32_t* col_idx, void* stream) {
  using namespace bsa::topk;
  // The argument checks of bsa_topk_pattern, then the scratch limit: all
  // before any CUDA call.
  if (!Q || !K || !row_ptr || !col_idx) return BSA_ERR_INVALID_ARG;
  if (BH < 1 || N < 1 || d < 1 || block_size < 1 || top_k < 0) return BSA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return BSA_ERR_INVALID_ARG;
  if (N % block_size != 0) return BSA_ERR_INVALID_ARG;
  const int M = N / block_size;
  if (d > kMaxD || M > kMaxM) return BSA_ERR_UNSUPPORTED;
  const size_t need = bsa_topk_workspace_bytes(BH, N, d, block_size);
  if (need > kStaticScratchBytes) return BSA_ERR_BUFFER_TOO_SMALL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
  void* scratch = static_scratch(dev);
  if (!scratch) return BSA_ERR_CUDA;
  return bsa_topk_pattern(Q, K, BH, N, d, block_size, top_k, causal, row_ptr, col_idx, scratch,
                          kStaticScratchBytes, stream);
}
