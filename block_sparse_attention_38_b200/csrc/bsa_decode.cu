// bsa_decode.cu -- one decode step of block-sparse attention over a KV cache.
//
// "Block Sparse Attention with Log-Linear Complexity" keeps the KV cache in
// the (B, H, N, D) layout of past_key_values (section 5.1) and claims the
// pattern cuts cache traffic at inference (section 1).  A decode step gives
// each (b, h) one new token at position t = seq_len[b] - 1, in block row
// i = t / bs; it attends to the cached tokens (up to t) of the blocks j <= i
// that CSR row i of head h lists, and optionally first appends its own k and
// v at cache row t.
//
// The work is a matrix-vector product streamed from HBM, so it runs on the
// CUDA cores, fed by TMA:
//   * one CTA per (b, h): a producer warp and NW consumer warps (3 for
//     d = 128, 4 for d = 64);
//   * the producer dedups the CSR row into a bitmap of blocks j <= i, splits
//     the blocks into units of 32 cache rows and TMA-loads each unit's K and
//     V rows (128-byte swizzle) into shared-memory stages;
//   * consumer warp w takes units w, w + NW, ... and owns the stages
//     w, w + NW, ... (its own ring of 2 or 3 stages, used in order, so that
//     the next unit's load overlaps the current unit's arithmetic, and so an
//     mbarrier phase it waits for is never two phases ahead of the last one
//     it consumed);
//   * lane l scores key l of a unit (the swizzle makes the 32 row reads
//     conflict-free; q is a shared-memory broadcast), then the warp
//     accumulates P . V with d/32 output columns per lane, in an online
//     softmax of its own; the warps' partial (m, l, o) are merged at the end.
// Two CTAs fit on an SM (at most about 100 KB of shared memory each), so every
// (b, h) of a batch of a few hundred is resident at once and the loads of
// all of them overlap.  Every wait is bounded: a wait that gives up sets
// BSA_STATUS_TIMEOUT and the CTA drains its copies and finishes.
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
namespace decode {

constexpr int kMaxM = 4096;
constexpr int kMaxConsumerWarps = 4;
constexpr int kStageBudget = 96 * 1024;
constexpr long long kWaitLimitCycles = 4000000000LL;  // ~2 s at 1.97 GHz

__device__ unsigned int g_decode_status;

constexpr int UK = 32;  // cache rows per unit: one key per lane

template <int D>
struct Cfg {
  static constexpr int ATOMS = D / 64;                          // 128-byte swizzle atoms per row
  static constexpr int ATOM_BYTES = UK * 128;                   // one TMA box: 32 rows x 128 bytes
  static constexpr int HALF = ATOMS * ATOM_BYTES;               // the K (or the V) rows of a unit
  static constexpr int STAGE = 2 * HALF;                        // 8 KB (d = 64) or 16 KB (d = 128)
  static constexpr int NW = D == 128 ? 3 : 4;                   // consumer warps
  static constexpr int THREADS = 32 * (NW + 1);                 // and one producer warp
  static constexpr int NSW = kStageBudget / (NW * STAGE);       // stages per consumer warp: 3 or 2
  static constexpr int NS = NW * NSW;                           // 12 or 6 stages
  static constexpr int CPL = D / 32;                            // output columns per lane
  static_assert(NSW >= 1 && NW <= kMaxConsumerWarps && NS <= 12, "stage ring");
  // unit u: consumer warp u % W, that warp's (u / W)-th unit
  __device__ static int stage(int u) {
    return u % NW + NW * ((u / NW) % NSW);
  }
  __device__ static uint32_t phase(int u) { return static_cast<uint32_t>(u / NW / NSW); }
};

struct Ctrl {
  uint64_t full[12];
  uint64_t empty[12];
  int nvalid[12];
  uint32_t bitmap[kMaxM / 32];
  int n_units;
  volatile int abort;
  alignas(16) float q[128];  // read as float4
  float part_m[kMaxConsumerWarps];
  float part_l[kMaxConsumerWarps];
  float part_o[kMaxConsumerWarps][128];
};

static_assert(offsetof(Ctrl, q) % 16 == 0, "q is read with 16-byte loads");
static_assert(sizeof(Ctrl) % 8 == 0, "mbarriers need 8-byte alignment");

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
        atomicOr(&g_decode_status, BSA_STATUS_TIMEOUT);
        return false;
      }
    }
  }
}

// Teardown: waits (bounded) for copies already issued, whatever the abort flag says.
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  for (uint32_t it = 0; !mbar_try_wait(bar, parity); ++it) {
    if ((it & 1023u) == 1023u && clock64() - t0 > kWaitLimitCycles) {
      atomicOr(&g_decode_status, BSA_STATUS_TIMEOUT);
      return;
    }
  }
}

// Orders this thread's generic-proxy global writes before later async-proxy
// (TMA) reads of the same addresses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ float bf16lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

struct Args {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int32_t* seq_len;
  __nv_bfloat16* O;
  float* LSE;
  int H, L, M, bs;
  float scale_log2;
};

template <int D>
__global__ void __launch_bounds__(Cfg<D>::THREADS, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                  const Args a) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Ctrl* ctl = reinterpret_cast<Ctrl*>(smem + C::NS * C::STAGE);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const long long bh = blockIdx.x;
  const int b = static_cast<int>(bh / a.H);
  const int h = static_cast<int>(bh - static_cast<long long>(b) * a.H);
  const int len = a.seq_len[b];
  const bool len_ok = len >= 1 && len <= a.L;
  const int t = len_ok ? len - 1 : 0;
  const int i = t / a.bs;

  if (warp == C::NW) {
    // ---------------------------------------------------------- producer setup
    if (lane == 0) {
      for (int s = 0; s < C::NS; ++s) {
        mbar_init(&ctl->full[s], 1);
        mbar_init(&ctl->empty[s], 1);
      }
      fence_mbar_init();
      ctl->abort = 0;
      if (!len_ok) atomicOr(&g_decode_status, BSA_STATUS_BAD_SEQ_LEN);
      prefetch_tensormap(&tk);
      prefetch_tensormap(&tv);
    }
    if (len_ok && a.k_new != nullptr && lane < D / 8) {
      // append: row t of this (b, h) gets the new token's k and v (16 bytes a lane)
      const long long row = (bh * a.L + t) * D + lane * 8;
      reinterpret_cast<uint4*>(a.k_cache + row)[0] =
          reinterpret_cast<const uint4*>(a.k_new + bh * D + lane * 8)[0];
      reinterpret_cast<uint4*>(a.v_cache + row)[0] =
          reinterpret_cast<const uint4*>(a.v_new + bh * D + lane * 8)[0];
      fence_proxy_async_global();
    }
    const int W = i / 32 + 1;
    for (int w = lane; w < W; w += 32) ctl->bitmap[w] = 0u;
    __syncwarp();
    int rp0 = 0, rp1 = 0;
    if (len_ok) {
      rp0 = a.row_ptr[static_cast<long long>(h) * a.M + i];
      rp1 = a.row_ptr[static_cast<long long>(h) * a.M + i + 1];
      if (rp0 < 0 || rp1 < rp0) {
        if (lane == 0) atomicOr(&g_decode_status, BSA_STATUS_BAD_ROW_PTR);
        rp0 = rp1 = 0;
      }
    }
    for (int e = rp0 + lane; e < rp1; e += 32) {
      const int j = a.col_idx[e];
      if (j < 0 || j >= a.M) {
        atomicOr(&g_decode_status, BSA_STATUS_BAD_COLUMN);
      } else if (j <= i) {
        atomicOr(&ctl->bitmap[j >> 5], 1u << (j & 31));
      }
    }
    __syncwarp();
    // units: UK-row pieces of every listed block j < i, and of the rows
    // i*bs .. t of block i
    int units = 0;
    for (int w = lane; w < W; w += 32) units += __popc(ctl->bitmap[w]);
    for (int o = 16; o > 0; o >>= 1) units += __shfl_xor_sync(0xffffffffu, units, o);
    if (lane == 0) {
      const bool diag = (ctl->bitmap[i >> 5] >> (i & 31)) & 1u;
      const int per_block = a.bs / UK;
      const int last = (t - i * a.bs + 1 + UK - 1) / UK;
      ctl->n_units = (units - (diag ? 1 : 0)) * per_block + (diag ? last : 0);
    }
  } else {
    for (int c = tid; c < D; c += C::NW * 32)
      ctl->q[c] = __bfloat162float(a.q[bh * D + c]);
  }
  __syncthreads();
  const int n_units = ctl->n_units;

  if (warp == C::NW) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      int u = 0;
      bool ok = true;
      const int W = i / 32 + 1;
      for (int w = 0; w < W && ok; ++w) {
        uint32_t bits = ctl->bitmap[w];
        while (bits != 0u && ok) {
          const int j = w * 32 + __ffs(bits) - 1;
          bits &= bits - 1;
          const int rows = j < i ? a.bs : t - i * a.bs + 1;
          for (int r0 = 0; r0 < rows; r0 += UK) {
            // the previous use of this stage is unit u - NS, of the same consumer warp
            const int s = C::stage(u);
            if (u >= C::NS && !wait_bounded(&ctl->empty[s], (C::phase(u) - 1) & 1, &ctl->abort)) {
              ok = false;
              break;
            }
            ctl->nvalid[s] = min(UK, rows - r0);
            unsigned char* st = smem + s * C::STAGE;
            mbar_arrive_expect_tx(&ctl->full[s], C::STAGE);
            const int row0 = j * a.bs + r0;
#pragma unroll
            for (int at = 0; at < C::ATOMS; ++at) {
              tma_load_3d(st + at * C::ATOM_BYTES, &tk, &ctl->full[s], at * 64, row0,
                          static_cast<int>(bh));
              tma_load_3d(st + C::HALF + at * C::ATOM_BYTES, &tv, &ctl->full[s], at * 64, row0,
                          static_cast<int>(bh));
            }
            ++u;
          }
        }
      }
      // Teardown: the last use of each stage must have landed before the CTA
      // ends (earlier uses were seen by their consumers before being refilled).
      for (int v = u > C::NS ? u - C::NS : 0; v < u; ++v)
        wait_drain(&ctl->full[C::stage(v)], C::phase(v) & 1);
    }
  } else {
    // ------------------------------------------------------------- consumers
    float m = -INFINITY;  // running max, log2 units (scores already scaled)
    float lsum = 0.f;     // this lane's share of the denominator
    float o[C::CPL];
#pragma unroll
    for (int c = 0; c < C::CPL; ++c) o[c] = 0.f;
    const float4* q4 = reinterpret_cast<const float4*>(ctl->q);

    for (int u = warp; u < n_units; u += C::NW) {
      const int s = C::stage(u);
      const bool got = wait_bounded(&ctl->full[s], C::phase(u) & 1, &ctl->abort);
      if (!__all_sync(0xffffffffu, got)) break;
      const int nv = ctl->nvalid[s];
      const unsigned char* Ks = smem + s * C::STAGE;
      const unsigned char* Vs = Ks + C::HALF;

      // score of key `lane`
      float sc = -INFINITY;
      if (lane < nv) {
        float acc = 0.f;
#pragma unroll
        for (int cc = 0; cc < D / 8; ++cc) {
          const int phys = (cc & 7) ^ (lane & 7);
          const uint4 kv = *reinterpret_cast<const uint4*>(Ks + (cc >> 3) * C::ATOM_BYTES +
                                                           lane * 128 + phys * 16);
          const float4 qa = q4[2 * cc], qb = q4[2 * cc + 1];
          acc = fmaf(qa.x, bf16lo(kv.x), acc);
          acc = fmaf(qa.y, bf16hi(kv.x), acc);
          acc = fmaf(qa.z, bf16lo(kv.y), acc);
          acc = fmaf(qa.w, bf16hi(kv.y), acc);
          acc = fmaf(qb.x, bf16lo(kv.z), acc);
          acc = fmaf(qb.y, bf16hi(kv.z), acc);
          acc = fmaf(qb.z, bf16lo(kv.w), acc);
          acc = fmaf(qb.w, bf16hi(kv.w), acc);
        }
        sc = acc * a.scale_log2;
      }
      float umax = sc;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        umax = fmaxf(umax, __shfl_xor_sync(0xffffffffu, umax, off));
      const float m_new = fmaxf(m, umax);  // finite: a unit holds at least one key
      const float alpha = ex2_approx(m - m_new);
      const float p = lane < nv ? ex2_approx(sc - m_new) : 0.f;
      lsum = lsum * alpha + p;
#pragma unroll
      for (int c = 0; c < C::CPL; ++c) o[c] *= alpha;
      m = m_new;

      // o += p . V over the unit's valid rows
      for (int k = 0; k < nv; ++k) {
        const float pk = __shfl_sync(0xffffffffu, p, k);
        const unsigned char* vrow = Vs + k * 128;
        if constexpr (C::CPL == 4) {
          const int c16 = lane >> 1;
          const uint2 vv = *reinterpret_cast<const uint2*>(
              vrow + (c16 >> 3) * C::ATOM_BYTES + (((c16 & 7) ^ (k & 7)) * 16) + (lane & 1) * 8);
          o[0] = fmaf(pk, bf16lo(vv.x), o[0]);
          o[1] = fmaf(pk, bf16hi(vv.x), o[1]);
          o[2] = fmaf(pk, bf16lo(vv.y), o[2]);
          o[3] = fmaf(pk, bf16hi(vv.y), o[3]);
        } else {
          const int c16 = lane >> 2;
          const uint32_t vv = *reinterpret_cast<const uint32_t*>(
              vrow + (((c16 & 7) ^ (k & 7)) * 16) + (lane & 3) * 4);
          o[0] = fmaf(pk, bf16lo(vv), o[0]);
          o[1] = fmaf(pk, bf16hi(vv), o[1]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->empty[s]);
    }

    for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
    if (lane == 0) {
      ctl->part_m[warp] = m;
      ctl->part_l[warp] = lsum;
    }
#pragma unroll
    for (int c = 0; c < C::CPL; ++c) ctl->part_o[warp][lane * C::CPL + c] = o[c];
  }
  __syncthreads();

  // ----------------------------------------------------------------- merge
  if (tid < D) {
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < C::NW; ++w) mx = fmaxf(mx, ctl->part_m[w]);
    float out = 0.f, den = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int w = 0; w < C::NW; ++w) {
        const float f = ex2_approx(ctl->part_m[w] - mx);
        den += ctl->part_l[w] * f;
        out += ctl->part_o[w][tid] * f;
      }
      out /= den;
    }
    a.O[bh * D + tid] = __float2bfloat16_rn(out);
    if (tid == 0)
      a.LSE[bh] = mx == -INFINITY ? -INFINITY : (mx + log2f(den)) * 0.6931471805599453f;
  }
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

// The cache [B*H, L, d] bf16 as a 3-D tensor; box = 64 columns x `rows` rows x 1.
bool make_cache_map(CUtensorMap* m, const void* base, long long BH, int L, int d, int rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(L) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
int launch(const Args& a, long long BH, const void* kc, const void* vc, cudaStream_t s) {
  using C = Cfg<D>;
  CUtensorMap tk, tv;
  if (!make_cache_map(&tk, kc, BH, a.L, D, UK) || !make_cache_map(&tv, vc, BH, a.L, D, UK))
    return BSA_ERR_CUDA;
  const int smem = C::NS * C::STAGE + static_cast<int>(sizeof(Ctrl)) + 1024;
  if (cudaFuncSetAttribute(decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess)
    return BSA_ERR_CUDA;
  decode_kernel<D><<<static_cast<unsigned>(BH), C::THREADS, smem, s>>>(tk, tv, a);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace decode
}  // namespace bsa

extern "C" int bsa_decode(const void* q, const void* k_new, const void* v_new, void* k_cache,
                          void* v_cache, const int32_t* row_ptr, const int32_t* col_idx,
                          const int32_t* seq_len, int B, int H, int L, int d, int block_size,
                          float scale, void* O, float* LSE, void* stream) {
  using namespace bsa::decode;
  if (!q || !k_cache || !v_cache || !row_ptr || !col_idx || !seq_len || !O || !LSE)
    return BSA_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return BSA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || L < 1 || d < 1 || block_size < 1) return BSA_ERR_INVALID_ARG;
  if (L % block_size != 0 || !std::isfinite(scale)) return BSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(O) ||
      (k_new && (!aligned16(k_new) || !aligned16(v_new))) ||
      (reinterpret_cast<uintptr_t>(LSE) & 3u) != 0)
    return BSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BSA_ERR_UNSUPPORTED;
  if (block_size != 32 && block_size != 64 && block_size != 128) return BSA_ERR_UNSUPPORTED;
  const int M = L / block_size;
  if (M > kMaxM) return BSA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  if (BH > 0x7fffffffLL || static_cast<long long>(H) * M + 1 > 0x7fffffffLL)
    return BSA_ERR_UNSUPPORTED;
  Args a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k_new = static_cast<const __nv_bfloat16*>(k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(v_new);
  a.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  a.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.seq_len = seq_len;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.LSE = LSE;
  a.H = H;
  a.L = L;
  a.M = M;
  a.bs = block_size;
  a.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch<64>(a, BH, k_cache, v_cache, s)
                 : launch<128>(a, BH, k_cache, v_cache, s);
}

extern "C" int bsa_decode_status(uint32_t* status, int clear) {
  if (!status) return BSA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return BSA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, bsa::decode::g_decode_status, sizeof(v)) != cudaSuccess)
    return BSA_ERR_CUDA;
  if (clear) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(bsa::decode::g_decode_status, &z, sizeof(z)) != cudaSuccess)
      return BSA_ERR_CUDA;
  }
  *status = v;
  return BSA_OK;
}
