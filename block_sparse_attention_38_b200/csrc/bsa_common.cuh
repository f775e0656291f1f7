// bsa_common.cuh -- definitions shared by the forward kernels: the device
// status word, the launch arguments, bounded mbarrier waits and a bitmap
// iterator.  Included once, by bsa_forward.cu (a single translation unit).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "bsa.h"
#include "sm100_ptx.cuh"

namespace bsa {


constexpr int kMaxM = 4096;                 // block rows supported per head
constexpr int kMaxBitmapWords = kMaxM / 32;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: O is rescaled only when the max grows by > 2^8
constexpr long long kWaitLimitCycles = 4000000000LL;  // ~2 s at 1.97 GHz: a longer wait is a hang

__device__ unsigned int g_status;

struct FwdArgs {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  __nv_bfloat16* O;
  float* LSE;
  int H, N, M, G, W;      // G = tiles per (b, h); W = 32-bit words per block-row bitmap
  long long num_tiles;
  float scale_log2;       // scale * log2(e)
  int causal;
  // Chunked tiles (optional): a long tile's key walk is cut into chunks that
  // run as separate work units; each chunk stores its unnormalised partial
  // result, and the last chunk to finish merges them.
  float* part_o;                  // [part_cap][D][128] fp32: O of a chunk before division by l
  float2* part_ml;                // [part_cap][128]: (running maximum m, log2 units; sum l)
  unsigned long long* part_cnt;   // [part_cap][4]: per warp, epoch << 8 | chunks arrived
  int part_cap;                   // chunk slots in the workspace; 0 = no tile is cut
  unsigned long long epoch;       // distinct for every launch (< 2^56)
};

struct AbortFlag {
  volatile int v;
};

// Bounded wait: true when the phase of parity `parity` has completed; false
// once about kWaitLimitCycles SM cycles have passed (>= 2 s at the B200's top
// clock) or when another warp has already given up.  The cycle counter is read
// only every 1024 polls so that a phase completing during the wait is seen
// within one try_wait.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, AbortFlag* ab) {
  if (mbar_try_wait(bar, parity)) return true;
  long long t0 = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 1023u) == 0) {
      if (ab->v) return false;
      const long long now = clock64();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kWaitLimitCycles) {
        ab->v = 1;
        atomicOr(&g_status, BSA_STATUS_TIMEOUT);
        return false;
      }
    }
  }
}

// Same, for teardown: ignores the abort flag (used to drain copies already in flight).
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  for (uint32_t it = 0; !mbar_try_wait(bar, parity); ++it) {
    if ((it & 1023u) == 1023u && clock64() - t0 > kWaitLimitCycles) {
      atomicOr(&g_status, BSA_STATUS_TIMEOUT);
      return;
    }
  }
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, AbortFlag* ab) {
  const bool ok = wait_bounded(bar, parity, ab);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ int union_count(const uint32_t* uni, int W) {
  int n = 0;
  for (int w = 0; w < W; ++w) n += __popc(uni[w]);
  return n;
}

// Walks the set bits of a bitmap in ascending order.
struct BitIter {
  const uint32_t* bits;
  int W, w;
  uint32_t cur;
  __device__ __forceinline__ BitIter(const uint32_t* b, int W_) : bits(b), W(W_), w(0), cur(b[0]) {}
  // Passes over the next k set bits (fewer if the map runs out first).
  __device__ __forceinline__ void skip(int k) {
    while (k > 0) {
      if (cur == 0) {
        if (++w >= W) return;
        cur = bits[w];
        continue;
      }
      const int c = __popc(cur);
      if (c <= k) {
        k -= c;
        cur = 0;
      } else {
        for (; k > 0; --k) cur &= cur - 1;
      }
    }
  }
  __device__ __forceinline__ int next() {
    while (cur == 0) {
      if (++w >= W) return -1;
      cur = bits[w];
    }
    const int b = __ffs(cur) - 1;
    cur &= cur - 1;
    return w * 32 + b;
  }
};


}  // namespace bsa
