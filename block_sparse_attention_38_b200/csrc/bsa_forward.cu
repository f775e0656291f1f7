// bsa_forward.cu -- host side of the block-sparse attention forward: argument
// validation, TMA descriptor encoding and the launch of the sm_100a two-slot
// kernel (one instantiation per block size and head dimension), plus the
// device status word.  The kernel lives in the headers this file includes;
// the library's other CUDA translation units are bsa_topk.cu, bsa_decode.cu
// and bsa_backward.cu.
#include <atomic>
#include <mutex>

#include "bsa_common.cuh"
#include "bsa_fwd_pp.cuh"

namespace bsa {

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

// [B*H, N, d] bf16 viewed as a 3-D tensor; box = 64 columns x `rows` rows x 1 head,
// 128-byte swizzle (the layout tcgen05 reads as K-major or MN-major SW128).
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
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DeviceInfo {
  int sms = 0;
};

std::mutex& device_mutex() {
  static std::mutex mu;
  return mu;
}

bool device_info(int dev, DeviceInfo* out) {
  static DeviceInfo cache[64];
  if (dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(device_mutex());
  DeviceInfo& di = cache[dev];
  if (di.sms == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return false;
    di.sms = sms;
  }
  *out = di;
  return true;
}

// Raises the dynamic shared-memory limit of the <BS, D, POS, CAUSAL> kernel
// on `dev` to `bytes` once per instantiation and device, under the device mutex.
template <int BS, int D, bool POS, bool CAUSAL>
bool ensure_smem_attr(int dev, int bytes) {
  static int set_bytes[64] = {};
  if (dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(device_mutex());
  if (set_bytes[dev] >= bytes) return true;
  if (cudaFuncSetAttribute(pp::fwd_kernel<BS, D, POS, CAUSAL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           bytes) != cudaSuccess)
    return false;
  set_bytes[dev] = bytes;
  return true;
}

// Workspace of the chunked tiles: the count words first (4 per chunk slot,
// kMaxVirt slots), then per chunk slot its (m, l) pairs and its O columns.
constexpr size_t kPartHeader = static_cast<size_t>(pp::kMaxVirt) * 4 * 8;
size_t part_slot_bytes(int d) { return 128 * 8 + 128 * static_cast<size_t>(d) * 4; }

std::atomic<unsigned long long>& launch_epoch() {
  static std::atomic<unsigned long long> e{1};
  return e;
}

template <int BS, int D>
int launch_fwd(const void* Q, const void* K, const void* V, const int32_t* row_ptr,
               const int32_t* col_idx, int B, int H, int N, float scale, int causal, void* O,
               float* LSE, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  using C = pp::Cfg<BS, D>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  DeviceInfo di;
  if (!device_info(dev, &di)) return BSA_ERR_CUDA;
  const long long BH = static_cast<long long>(B) * H;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, Q, BH, N, D, C::TM) || !make_map(&tk, K, BH, N, D, BS) ||
      !make_map(&tv, V, BH, N, D, BS))
    return BSA_ERR_CUDA;
  FwdArgs a;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.LSE = LSE;
  a.H = H;
  a.N = N;
  a.M = N / BS;
  a.G = (a.M + C::R - 1) / C::R;
  a.W = (a.M + 31) / 32;
  a.num_tiles = BH * a.G;
  a.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  // The kernel scales masked keys (+-inf) by the scale; a zero scale becomes
  // the smallest normal float, which leaves every unmasked score at 0 to
  // within fp32 rounding and sends masked ones to -inf.
  if (a.scale_log2 == 0.f) a.scale_log2 = 1.17549435e-38f;
  a.causal = causal;
  a.part_o = nullptr;
  a.part_ml = nullptr;
  a.part_cnt = nullptr;
  a.part_cap = 0;
  a.epoch = launch_epoch().fetch_add(1) & ((1ull << 56) - 1);
  if (workspace && workspace_bytes >= kPartHeader + part_slot_bytes(D)) {
    const size_t cap = (workspace_bytes - kPartHeader) / part_slot_bytes(D);
    a.part_cap = static_cast<int>(cap < static_cast<size_t>(pp::kMaxVirt) ? cap : pp::kMaxVirt);
    uint8_t* w = static_cast<uint8_t*>(workspace);
    a.part_cnt = reinterpret_cast<unsigned long long*>(w);
    a.part_ml = reinterpret_cast<float2*>(w + kPartHeader);
    a.part_o = reinterpret_cast<float*>(w + kPartHeader + static_cast<size_t>(a.part_cap) * 128 * 8);
  }
  // stages, control block, the tile-bitmap buffers, and 1024 bytes of alignment slack
  const int smem = C::OFF_CTRL + static_cast<int>(sizeof(pp::Ctrl)) +
                   pp::kSlots * pp::kTiRing * pp::bitmap_words<BS>(a.W) * 4 + 1024;
  long long grid = a.num_tiles < di.sms ? a.num_tiles : di.sms;
  if (grid > pp::kMaxGrid) grid = pp::kMaxGrid;
  // One instantiation per sign of the scale and per causal flag: each kernel
  // carries only the row-maximum code (maximum or minimum of the raw scores)
  // and the diagonal masking it runs.
  const unsigned g = static_cast<unsigned>(grid);
  const bool pos = a.scale_log2 > 0.f;
  if (pos && causal) {
    if (!ensure_smem_attr<BS, D, true, true>(dev, smem)) return BSA_ERR_CUDA;
    pp::fwd_kernel<BS, D, true, true><<<g, pp::kThreads, smem, stream>>>(tq, tk, tv, a);
  } else if (pos) {
    if (!ensure_smem_attr<BS, D, true, false>(dev, smem)) return BSA_ERR_CUDA;
    pp::fwd_kernel<BS, D, true, false><<<g, pp::kThreads, smem, stream>>>(tq, tk, tv, a);
  } else if (causal) {
    if (!ensure_smem_attr<BS, D, false, true>(dev, smem)) return BSA_ERR_CUDA;
    pp::fwd_kernel<BS, D, false, true><<<g, pp::kThreads, smem, stream>>>(tq, tk, tv, a);
  } else {
    if (!ensure_smem_attr<BS, D, false, false>(dev, smem)) return BSA_ERR_CUDA;
    pp::fwd_kernel<BS, D, false, false><<<g, pp::kThreads, smem, stream>>>(tq, tk, tv, a);
  }
  if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  return BSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace bsa

extern "C" size_t bsa_forward_workspace_bytes(int d) {
  using namespace bsa;
  if (d != 64 && d != 128) return 0;
  return kPartHeader + static_cast<size_t>(pp::kMaxVirt) * part_slot_bytes(d);
}

extern "C" int bsa_forward(const void* Q, const void* K, const void* V, const int32_t* row_ptr,
                           const int32_t* col_idx, int B, int H, int N, int d, int block_size,
                           float scale, int causal, void* O, float* LSE, void* stream) {
  return bsa_forward_ws(Q, K, V, row_ptr, col_idx, B, H, N, d, block_size, scale, causal, O, LSE,
                        nullptr, 0, stream);
}

extern "C" int bsa_forward_ws(const void* Q, const void* K, const void* V, const int32_t* row_ptr,
                              const int32_t* col_idx, int B, int H, int N, int d, int block_size,
                              float scale, int causal, void* O, float* LSE, void* workspace,
                              size_t workspace_bytes, void* stream) {
  using namespace bsa;
  if (!Q || !K || !V || !row_ptr || !col_idx || !O || !LSE) return BSA_ERR_INVALID_ARG;
  if (workspace && !aligned16(workspace)) return BSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || block_size <= 0) return BSA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return BSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return BSA_ERR_INVALID_ARG;
  if (N % block_size != 0) return BSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE))
    return BSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BSA_ERR_UNSUPPORTED;
  if (block_size != 32 && block_size != 64 && block_size != 128) return BSA_ERR_UNSUPPORTED;
  if (N / block_size > kMaxM) return BSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > 2147483647LL) return BSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(H) * (N / block_size) + 1 > 2147483647LL) return BSA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (block_size * 1000 + d) {
    case 32064: return launch_fwd<32, 64>(Q, K, V, row_ptr, col_idx, B, H, N, scale, causal, O, LSE, workspace, workspace_bytes, s);
    case 32128: return launch_fwd<32, 128>(Q, K, V, row_ptr, col_idx, B, H, N, scale, causal, O, LSE, workspace, workspace_bytes, s);
    case 64064: return launch_fwd<64, 64>(Q, K, V, row_ptr, col_idx, B, H, N, scale, causal, O, LSE, workspace, workspace_bytes, s);
    case 64128: return launch_fwd<64, 128>(Q, K, V, row_ptr, col_idx, B, H, N, scale, causal, O, LSE, workspace, workspace_bytes, s);
    case 128064: return launch_fwd<128, 64>(Q, K, V, row_ptr, col_idx, B, H, N, scale, causal, O, LSE, workspace, workspace_bytes, s);
    case 128128: return launch_fwd<128, 128>(Q, K, V, row_ptr, col_idx, B, H, N, scale, causal, O, LSE, workspace, workspace_bytes, s);
    default: return BSA_ERR_UNSUPPORTED;
  }
}

extern "C" int bsa_device_status(uint32_t* status, int clear) {
  using namespace bsa;
  if (!status) return BSA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return BSA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return BSA_ERR_CUDA;
  *status = v;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return BSA_ERR_CUDA;
  }
  return BSA_OK;
}
