// bsa_fwd_keys.cuh -- key-tile forward kernel for 32-token blocks.
//
// With 32-token blocks a block row holds only 32 queries, a quarter of the
// 128-row M dimension of a single-CTA tcgen05.mma.  The columns of one block
// row differ from those of its neighbours (log-stride blocks rarely
// coincide), so a tile of four block rows would compute their union, about
// 2.5 times the useful work.  This kernel puts the *keys* on M instead:
//
//   tile  = one block row (b, h, r): 32 queries and its L column blocks;
//   chunk = 4 of those column blocks gathered into 128 key rows;
//   S^T   = K_chunk Q^T          (M=128 keys, N=32 queries, K=d) -> TMEM;
//   O^T  += V_chunk^T P^T        (M=d rows, N=32 queries, K=128 keys) -> TMEM.
//
// Thread t of a softmax warpgroup owns key row t of a chunk and reads its 32
// query scores with one tcgen05.ld.  The softmax is restricted to the
// connected key blocks ("Block Sparse Attention with Log-Linear Complexity",
// section 3.3: the denominator sums only over them).  It runs in one pass per
// chunk with a lazily updated maximum: p = 2^(s - m) with the current
// per-query maximum m as long as no score exceeds m by more than 2^8 (a
// warpgroup-wide vote per chunk); otherwise -- always on a row's first chunk
// -- the exact per-query maximum is formed by a warp transpose-reduction (31
// shuffles for 32 queries) and a 4-warp exchange in shared memory, and O^T
// and the row sums are rescaled.  Row sums are kept in fp32 per thread and
// reduced once per tile.  For d = 64 the O^T MMA still uses M = 128 (the
// single-CTA shape whose TMEM layout is one row per lane): the upper 64 rows
// of its A operand are a constant zero tile and rows 64..127 of O^T are
// ignored.
//
// A CTA runs NWG independent pipelines.  Each has a softmax warpgroup (whose
// thread 0 also issues that pipeline's MMAs) and two copy warps: one builds
// the tile's column bitmap and gathers Q and the K chunks, the other gathers
// the V chunks.  The copies are 16-byte cp.async transfers written straight
// into the 128-byte-swizzled layout the MMA reads (many small copies in
// flight reach a far higher gather rate than bulk tensor copies issued from
// one thread, which are serviced one after another); a missing block of a
// partial chunk is zero-filled.  Completion is signalled per stage with
// cp.async.mbarrier.arrive.noinc, and the MMA-issuing thread fences the
// generic-proxy writes after its barrier wait.  The copy warps never fence
// (a proxy fence waits for the issuing thread's own copies in flight), and
// the threads that fence never have copies in flight.  The copy warps give up
// registers (setmaxnreg) to the softmax warpgroups.
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace keys {

constexpr float kLazyMaxSlack = 8.0f;  // log2 units: P may reach 2^8 before a rescale

template <int D>
struct Cfg {
  static constexpr int NWG = (D == 64) ? 2 : 1;  // independent pipelines per CTA
  static constexpr int THREADS = 128 * NWG + 128;  // + one warpgroup of copy warps
  static constexpr int COPY_WG = NWG;            // warpgroup index of the copy warps
  static constexpr int Q_BYTES = 32 * D * 2;     // 32 query rows
  static constexpr int QATOM = 32 * 128;         // 32 rows x 128 B
  static constexpr int CH_BYTES = 128 * D * 2;   // one K or V chunk: 128 key rows
  static constexpr int CHATOM = 128 * 128;       // 128 rows x 128 B
  static constexpr int NKS = 3;                  // K stages per pipeline
  static constexpr int NVS = 2;                  // V stages per pipeline
  static constexpr int P_BYTES = 128 * 32 * 2;   // P^T of a chunk: 128 keys x 32 queries
  static constexpr bool PAD_A = (D == 64);       // zero upper half of the O^T A operand
  // per-pipeline layout (offsets from the pipeline's base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NKS * CH_BYTES;
  static constexpr int OFF_P = OFF_V + NVS * CH_BYTES;
  static constexpr int WG_BYTES = OFF_P + 2 * P_BYTES;
  // CTA layout
  static constexpr int OFF_PAD = NWG * WG_BYTES;
  static constexpr int OFF_CTRL = OFF_PAD + (PAD_A ? CHATOM : 0);
  static constexpr uint32_t TMEM_COLS = 128 * NWG;  // per pipeline: 2 S^T chunks + O^T
  // register split: the copy warpgroup shrinks, the softmax warpgroups grow
  static constexpr int REGS_AT_LAUNCH = 65536 / THREADS / 8 * 8;
  static constexpr int REGS_COPY = 80;
  static constexpr int REGS_SOFTMAX =
      ((REGS_AT_LAUNCH * THREADS - REGS_COPY * 128) / (128 * NWG)) / 8 * 8 > 240
          ? 240
          : ((REGS_AT_LAUNCH * THREADS - REGS_COPY * 128) / (128 * NWG)) / 8 * 8;
  static_assert(REGS_SOFTMAX * 128 * NWG + REGS_COPY * 128 <= REGS_AT_LAUNCH * THREADS,
                "register split exceeds the launch's registers");
  static_assert(Q_BYTES % 1024 == 0 && CH_BYTES % 1024 == 0 && WG_BYTES % 1024 == 0, "alignment");
};

struct alignas(16) PipeCtrl {
  uint64_t bm_full[2], bm_empty[2];  // column bitmap written / read by all its readers
  uint64_t qfull, qempty;            // Q copied (32 arrivals) / last QK of the tile done
  uint64_t kfull[3], kempty[3];      // K stage copied (32 arrivals) / its QK done
  uint64_t vfull[2], vempty[2];      // V stage copied (32 arrivals) / its PV done
  uint64_t sbar[2];                  // S^T chunk ready (tcgen05.commit)
  uint64_t obar;                     // one PV product completed (tcgen05.commit)
  uint64_t fbar;                     // every MMA of this pipeline completed (teardown)
  uint32_t bitmap[2][kMaxBitmapWords];
  alignas(16) float red[4][32];
  alignas(16) float bcast[32];  // read back as float4
  alignas(16) float lsum[32];   // read back as float4
};

struct Ctrl {
  PipeCtrl pipe[2];
  uint32_t tmem_base;
  AbortFlag abort;
};

// Lane L ends with op over the 32 lanes of v[L] (v is consumed).
template <typename Op>
__device__ __forceinline__ float transpose_reduce(float (&v)[32], Op op) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, off);
      v[i] = op(keep, recv);
    }
  }
  return v[0];
}

// OR of `pred` over the 128 threads that meet at named barrier `id` (warp
// reconverged first; non-aligned form, as for named_bar).
__device__ __forceinline__ bool named_bar_or(int id, bool pred) {
  __syncwarp();
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "barrier.red.or.pred p, %2, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// One copy warp gathers a chunk (4 blocks of 32 rows) into `stage` with the
// 128-byte swizzle: 16-byte piece p of row r of an atom sits at piece
// p ^ (r & 7).  Lane l copies piece l % PPR of rows l / PPR + k * (32 / PPR),
// so a warp instruction moves 512 contiguous bytes and, per lane, the source
// and destination of consecutive copies are a fixed stride apart; the swizzle
// term repeats every 8 rows, so its few distinct values are precomputed once
// per lane (GatherPlan).  blocks[b] < 0 marks a missing block (zero-filled).
template <int D>
struct GatherPlan {
  static constexpr int PPR = D / 8;             // 16-byte pieces per row
  static constexpr int RPI = 32 / PPR;          // rows covered by one warp instruction
  static constexpr int ITERS = 32 / RPI;        // instructions per block
  static constexpr int NSW = 8 / RPI;           // distinct (row & 7) patterns across iterations
  int src;                                      // element offset of this lane's first piece
  uint32_t dst[NSW];                            // byte offset inside a block, iteration i % NSW
  __device__ __forceinline__ explicit GatherPlan(int lane) {
    const int r0 = lane / PPR, pc = lane % PPR;
    src = r0 * D + pc * 8;
#pragma unroll
    for (int v = 0; v < NSW; ++v) {
      const int r = v * RPI + r0;               // row of iteration v (mod 8)
      dst[v] = (pc >> 3) * (128 * 128) + r * 128 + (((pc & 7) ^ (r & 7)) << 4);
    }
  }
};

template <int D>
__device__ __forceinline__ void gather_chunk(uint32_t stage, const __nv_bfloat16* head,
                                             const int (&blocks)[4], const GatherPlan<D>& g) {
  using G = GatherPlan<D>;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const int j = blocks[b];
    const uint32_t bytes = j >= 0 ? 16u : 0u;
    const __nv_bfloat16* src = head + static_cast<long long>(j >= 0 ? j : 0) * 32 * D + g.src;
    const uint32_t dst = stage + b * 4096;
#pragma unroll
    for (int i = 0; i < G::ITERS; ++i)
      cp_async_16(dst + (i / G::NSW) * (8 * 128) + g.dst[i % G::NSW], src + i * G::RPI * D, bytes);
  }
}

struct TileRef {
  long long bh;
  int r, h;
};

__device__ __forceinline__ TileRef tile_ref(const FwdArgs& a, long long tile) {
  TileRef t;
  t.bh = tile / a.M;
  t.r = static_cast<int>(tile - t.bh * a.M);
  t.h = static_cast<int>(t.bh % a.H);
  return t;
}

__device__ __forceinline__ int popcount_words(const uint32_t* w, int W) {
  int n = 0;
  for (int i = 0; i < W; ++i) n += __popc(w[i]);
  return n;
}

// ------------------------------------------------------------ copy warps
// K warp: builds each tile's column bitmap, then gathers Q and the K chunks.
template <int D>
__device__ void copy_warp_qk(const FwdArgs& a, uint8_t* base, PipeCtrl* pc, AbortFlag* ab, int wg) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  const uint32_t q_s = smem_u32(base + C::OFF_Q);
  const uint32_t k_s = smem_u32(base + C::OFF_K);
  const GatherPlan<D> plan(lane);
  uint32_t k_issued = 0, q_issued = 0;
  bool ok = true;
  const long long stride = static_cast<long long>(gridDim.x) * C::NWG;
  int k = 0;
  for (long long tile = static_cast<long long>(blockIdx.x) * C::NWG + wg; ok && tile < a.num_tiles;
       tile += stride, ++k) {
    const int slot = k & 1;
    int w_ok = 1;
    if (lane == 0) w_ok = wait_bounded(&pc->bm_empty[slot], ((k >> 1) & 1) ^ 1, ab);
    if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
    uint32_t* bm = pc->bitmap[slot];
    for (int w = lane; w < a.W; w += 32) bm[w] = 0u;
    __syncwarp();
    const TileRef t = tile_ref(a, tile);
    const int beg = __ldg(a.row_ptr + (static_cast<long long>(t.h) * a.M + t.r));
    const int end = __ldg(a.row_ptr + (static_cast<long long>(t.h) * a.M + t.r + 1));
    if (end < beg) {
      if (lane == 0) atomicOr(&g_status, BSA_STATUS_BAD_ROW_PTR);
    } else {
      for (int p = beg + lane; p < end; p += 32) {
        const int j = __ldg(a.col_idx + p);
        if (j < 0 || j >= a.M) {
          atomicOr(&g_status, BSA_STATUS_BAD_COLUMN);
          continue;
        }
        if (a.causal && j > t.r) continue;  // wholly above the diagonal: no allowed key
        atomicOr(&bm[j >> 5], 1u << (j & 31));
      }
    }
    __threadfence_block();
    __syncwarp();
    if (lane == 0) mbar_arrive(&pc->bm_full[slot]);
    const int L = popcount_words(bm, a.W);
    if (L == 0) continue;
    const __nv_bfloat16* khead = a.K + t.bh * static_cast<long long>(a.N) * D;
    // Q: 32 rows, 128-byte swizzle
    if (lane == 0) w_ok = wait_bounded(&pc->qempty, (q_issued & 1) ^ 1, ab);
    if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
    {
      const __nv_bfloat16* qsrc = a.Q + (t.bh * a.N + static_cast<long long>(t.r) * 32) * D;
      for (int p = lane; p < 32 * D / 8; p += 32) {
        const int rr = p / (D / 8), pp = p % (D / 8);
        cp_async_16(q_s + (pp >> 3) * C::QATOM + rr * 128 + (((pp & 7) ^ (rr & 7)) << 4),
                    qsrc + rr * D + pp * 8, 16u);
      }
      cp_async_arrive_noinc(&pc->qfull);
      ++q_issued;
    }
    BitIter it(bm, a.W);
    const int nch = (L + 3) / 4;
    for (int c = 0; c < nch; ++c) {
      int blk[4];
      for (int b = 0; b < 4; ++b) blk[b] = it.next();
      const uint32_t s = k_issued % C::NKS;
      if (lane == 0) w_ok = wait_bounded(&pc->kempty[s], ((k_issued / C::NKS) & 1) ^ 1, ab);
      if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
      gather_chunk<D>(k_s + s * C::CH_BYTES, khead, blk, plan);
      cp_async_arrive_noinc(&pc->kfull[s]);
      ++k_issued;
    }
  }
  cp_async_wait<0>();
  __syncwarp();
}

// V warp: gathers the V chunks of each tile.
template <int D>
__device__ void copy_warp_v(const FwdArgs& a, uint8_t* base, PipeCtrl* pc, AbortFlag* ab, int wg) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  const uint32_t v_s = smem_u32(base + C::OFF_V);
  const GatherPlan<D> plan(lane);
  uint32_t v_issued = 0;
  bool ok = true;
  const long long stride = static_cast<long long>(gridDim.x) * C::NWG;
  int k = 0;
  for (long long tile = static_cast<long long>(blockIdx.x) * C::NWG + wg; ok && tile < a.num_tiles;
       tile += stride, ++k) {
    const int slot = k & 1;
    int w_ok = 1;
    if (lane == 0) w_ok = wait_bounded(&pc->bm_full[slot], (k >> 1) & 1, ab);
    if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
    const uint32_t* bm = pc->bitmap[slot];
    const TileRef t = tile_ref(a, tile);
    const __nv_bfloat16* vhead = a.V + t.bh * static_cast<long long>(a.N) * D;
    const int nch = (popcount_words(bm, a.W) + 3) / 4;
    BitIter it(bm, a.W);
    for (int c = 0; c < nch; ++c) {
      int blk[4];
      for (int b = 0; b < 4; ++b) blk[b] = it.next();
      const uint32_t s = v_issued % C::NVS;
      if (lane == 0) w_ok = wait_bounded(&pc->vempty[s], ((v_issued / C::NVS) & 1) ^ 1, ab);
      if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
      gather_chunk<D>(v_s + s * C::CH_BYTES, vhead, blk, plan);
      cp_async_arrive_noinc(&pc->vfull[s]);
      ++v_issued;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&pc->bm_empty[slot]);
  }
  cp_async_wait<0>();
  __syncwarp();
}

// ------------------------------------------------------- softmax warpgroup
template <int D>
__device__ void softmax_wg(const FwdArgs& a, uint8_t* smem, Ctrl* ctl, uint32_t tmem_base, int wg) {
  using C = Cfg<D>;
  constexpr float kNegInf = -INFINITY;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 32, false, false);  // K, Q: K-major
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 32, true, true);    // V^T, P^T: MN-major
  PipeCtrl* pc = &ctl->pipe[wg];
  AbortFlag* ab = &ctl->abort;
  const int tid = threadIdx.x & 127;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int bar_id = 1 + wg;
  uint8_t* base = smem + wg * C::WG_BYTES;
  const uint32_t q_s = smem_u32(base + C::OFF_Q);
  const uint32_t k_s = smem_u32(base + C::OFF_K);
  const uint32_t v_s = smem_u32(base + C::OFF_V);
  const uint32_t p_s = smem_u32(base + C::OFF_P);
  const uint32_t pad_s = smem_u32(smem + C::OFF_PAD);
  const uint32_t tmem = tmem_base + wg * 128;
  const uint32_t t_lane = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t s_col = tmem + t_lane;       // S^T chunk buffers at +0 and +32
  const uint32_t o_col = tmem + 64 + t_lane;  // O^T
  const float scale_log2 = a.scale_log2;
  const int causal = a.causal;
  const int W = a.W, N = a.N;

  // running counters: barrier phases continue across tiles
  uint32_t k_used = 0, v_used = 0, q_used = 0;
  uint32_t s_uses[2] = {0, 0};
  uint32_t pv_issued = 0, pv_seen = 0;
  bool ok = true;

  // all 128 threads agree: true iff every one of them passes `mine`
  auto all_ok = [&](bool mine) { return !named_bar_or(bar_id, !mine); };
  // The first `count` PVs of this pipeline completed.  Callers keep `count`
  // within one of the PVs issued: obar is one barrier whose phases are told
  // apart by parity, so at most one of its completions may go unobserved.
  auto ensure_pv_done = [&](uint32_t count) -> bool {
    bool good = true;
    while (good && pv_seen < count) {
      good = wait_bounded(&pc->obar, pv_seen & 1, ab);
      ++pv_seen;
    }
    return good;
  };
  // thread 0: S^T[sb] = K Q^T for the next K chunk
  auto issue_qk = [&](int sb, bool last) -> bool {
    const uint32_t ks = k_used % C::NKS;
    if (!wait_bounded(&pc->kfull[ks], (k_used / C::NKS) & 1, ab)) return false;
    fence_proxy_async_smem();  // the copy warp's writes, seen through the barrier
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t ad =
          sdesc_sw128(k_s + ks * C::CH_BYTES + (kk >> 2) * C::CHATOM + (kk & 3) * 32, 16, 1024);
      const uint64_t bd = sdesc_sw128(q_s + (kk >> 2) * C::QATOM + (kk & 3) * 32, 16, 1024);
      umma_bf16_ss(tmem + sb * 32, ad, bd, kIdescQK, kk > 0 ? 1u : 0u);
    }
    umma_commit(&pc->kempty[ks]);
    umma_commit(&pc->sbar[sb]);
    if (last) umma_commit(&pc->qempty);
    return true;
  };

  const long long stride = static_cast<long long>(gridDim.x) * C::NWG;
  int k = 0;
  for (long long tile = static_cast<long long>(blockIdx.x) * C::NWG + wg; ok && tile < a.num_tiles;
       tile += stride, ++k) {
    const int slot = k & 1;
    const TileRef t = tile_ref(a, tile);
    // ---- the tile's columns
    if (!(ok = all_ok(wait_bounded(&pc->bm_full[slot], (k >> 1) & 1, ab)))) break;
    const uint32_t* bm = pc->bitmap[slot];
    const int L = popcount_words(bm, W);
    int diag_pos = -1;
    if (causal && ((bm[t.r >> 5] >> (t.r & 31)) & 1u)) {
      diag_pos = 0;
      for (int w = 0; w < (t.r >> 5); ++w) diag_pos += __popc(bm[w]);
      diag_pos += __popc(bm[t.r >> 5] & ((1u << (t.r & 31)) - 1u));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&pc->bm_empty[slot]);
    const long long row0 = t.bh * N + static_cast<long long>(t.r) * 32;  // first query row
    if (L == 0) {  // no key at all: O = 0, LSE = -inf
      uint4* o = reinterpret_cast<uint4*>(a.O + row0 * D);
      for (int i = tid; i < 32 * D / 8; i += 128) o[i] = make_uint4(0u, 0u, 0u, 0u);
      if (warp == 0) a.LSE[row0 + lane] = kNegInf;
      continue;
    }
    const int nch = (L + 3) / 4;

    bool mine = true;
    if (tid == 0) {
      mine = wait_bounded(&pc->qfull, q_used & 1, ab) && issue_qk(0, nch == 1);
    }
    ++q_used;
    ++k_used;

    float mu[32];     // running max per query (log2 units of the scaled score)
    float lpart[32];  // this thread's partial row sums
    float m_own = kNegInf;  // running max of query `lane`
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      mu[q] = kNegInf;
      lpart[q] = 0.f;
    }
    const uint32_t pv_base = pv_issued;

    for (int c = 0; c < nch; ++c) {
      const int sb = c & 1;
      // ---- S^T of chunk c ready; thread 0 starts QK of chunk c + 1 at once
      mine = mine && wait_bounded(&pc->sbar[sb], s_uses[sb] & 1, ab);
      ++s_uses[sb];
      if (tid == 0 && mine && c + 1 < nch) mine = issue_qk(sb ^ 1, c + 2 == nch);
      if (c + 1 < nch) ++k_used;
      if (!(ok = all_ok(mine))) break;
      tc_fence_after();

      // ---- scores of this thread's key row for the 32 queries
      const int blk_slot = 4 * c + warp;  // block slot held by this warp
      const bool valid = blk_slot < L;
      const bool diag = (blk_slot == diag_pos);
      float x[32];
      if (valid) {
        uint32_t u[32];
        tmem_ld32(s_col + sb * 32, u);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const float v = __uint_as_float(u[q]) * scale_log2;
          x[q] = (diag && lane > q) ? kNegInf : v;
        }
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) x[q] = kNegInf;
      }
      tc_fence_before();

      // ---- lazy maximum: exact update only when a score outgrows it by > 2^8
      bool viol = false;
#pragma unroll
      for (int q = 0; q < 32; ++q) viol |= (x[q] > mu[q] + kLazyMaxSlack);
      if (named_bar_or(bar_id, viol)) {
        float mx[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) mx[q] = x[q];
        const float wmax = transpose_reduce(mx, [](float p, float s) { return fmaxf(p, s); });
        pc->red[warp][lane] = wmax;
        named_bar(bar_id, 128);
        const float gmax = fmaxf(fmaxf(pc->red[0][lane], pc->red[1][lane]),
                                 fmaxf(pc->red[2][lane], pc->red[3][lane]));
        m_own = fmaxf(m_own, gmax);
        if (warp == 0) pc->bcast[lane] = m_own;
        named_bar(bar_id, 128);
        float mnew[32];
#pragma unroll
        for (int q = 0; q < 32; q += 4) {
          const float4 t4 = *reinterpret_cast<const float4*>(&pc->bcast[q]);
          mnew[q] = t4.x;
          mnew[q + 1] = t4.y;
          mnew[q + 2] = t4.z;
          mnew[q + 3] = t4.w;
        }
        if (c > 0) {  // rescale what the earlier chunks accumulated
          if (!(ok = all_ok(ensure_pv_done(pv_base + c)))) break;
          tc_fence_after();
          uint32_t u[32];
          tmem_ld32(o_col, u);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const float f = (mu[q] == kNegInf) ? 0.f : ex2_approx(mu[q] - mnew[q]);
            u[q] = __float_as_uint(__uint_as_float(u[q]) * f);
            lpart[q] *= f;
          }
          tmem_st32(o_col, u);
          tmem_wait_st();
        }
#pragma unroll
        for (int q = 0; q < 32; ++q) mu[q] = mnew[q];
      }

      // ---- P^T = 2^(s - max) in bf16 into buffer sb.  PV(c - 1) is observed
      // here every iteration (see ensure_pv_done); that also frees buffer sb,
      // last read by PV(c - 2).
      if (c >= 1 && !(ok = all_ok(ensure_pv_done(pv_base + c)))) break;
      if (valid) {
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 32; q += 2) {
          const float p0 = ex2_approx(x[q] - (mu[q] == kNegInf ? 0.f : mu[q]));
          const float p1 = ex2_approx(x[q + 1] - (mu[q + 1] == kNegInf ? 0.f : mu[q + 1]));
          lpart[q] += p0;
          lpart[q + 1] += p1;
          pk[q >> 1] = pack_bf16x2(p0, p1);
        }
        const uint32_t rowp = p_s + sb * C::P_BYTES + tid * 64;  // 64-byte swizzle
        const uint32_t sw = (tid >> 1) & 3;
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16)
          st_shared_v4(rowp + ((c16 ^ sw) << 4), pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2],
                       pk[4 * c16 + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();

      // ---- PV of chunk c (thread 0 issues after every P^T row is written)
      named_bar(bar_id, 128);
      mine = true;
      if (tid == 0) {
        const uint32_t vs = v_used % C::NVS;
        mine = wait_bounded(&pc->vfull[vs], (v_used / C::NVS) & 1, ab);
        if (mine) {
          fence_proxy_async_smem();  // the copy warp's writes, seen through the barrier
          tc_fence_after();
          const uint32_t vstage = v_s + vs * C::CH_BYTES;
          const uint32_t lbo = C::PAD_A ? (pad_s - vstage) : static_cast<uint32_t>(C::CHATOM);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {  // 128 keys, 16 per MMA
            const uint64_t ad = sdesc(vstage + kk * 2048, lbo, 1024, kLayoutSW128);
            const uint64_t bd = sdesc(p_s + sb * C::P_BYTES + kk * 1024, C::P_BYTES, 512, kLayoutSW64);
            umma_bf16_ss(tmem + 64, ad, bd, kIdescPV, (c == 0 && kk == 0) ? 0u : 1u);
          }
          umma_commit(&pc->vempty[vs]);
          umma_commit(&pc->obar);
        }
      }
      ++v_used;
      ++pv_issued;
      if (!(ok = all_ok(mine))) break;
      mine = true;
    }
    if (!ok) break;

    // ---- epilogue: O = O^T / l, LSE = (max + log2 l) ln 2
    if (!(ok = all_ok(ensure_pv_done(pv_base + nch)))) break;
    tc_fence_after();
    uint32_t u[32];
    tmem_ld32(o_col, u);
    tmem_wait_ld();
    tc_fence_before();
    const float wsum = transpose_reduce(lpart, [](float p, float s) { return p + s; });
    pc->red[warp][lane] = wsum;
    named_bar(bar_id, 128);
    if (warp == 0)
      pc->lsum[lane] = (pc->red[0][lane] + pc->red[1][lane]) + (pc->red[2][lane] + pc->red[3][lane]);
    named_bar(bar_id, 128);
    if (warp < D / 32) {
      __nv_bfloat16* orow = a.O + row0 * D + tid;  // O^T row = head-dim index
#pragma unroll
      for (int q = 0; q < 32; q += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(&pc->lsum[q]);
        const float ls[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float inv = ls[i] > 0.f ? 1.f / ls[i] : 0.f;
          orow[static_cast<long long>(q + i) * D] =
              __float2bfloat16_rn(__uint_as_float(u[q + i]) * inv);
        }
      }
    }
    if (warp == 3) {
      const float l = pc->lsum[lane];
      a.LSE[row0 + lane] = l > 0.f ? (m_own + __log2f(l)) * 0.69314718055994531f : kNegInf;
    }
  }
  // teardown: every MMA of this pipeline completes before the CTA ends
  if (tid == 0) {
    umma_commit(&pc->fbar);
    wait_drain(&pc->fbar, 0);
  }
  __syncwarp();
}

template <int D>
__global__ void __launch_bounds__(Cfg<D>::THREADS, 1) fwd_kernel(const FwdArgs args) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Ctrl* ctl = reinterpret_cast<Ctrl*>(smem + C::OFF_CTRL);
  const int warp = threadIdx.x >> 5;
  const int wgi = warp >> 2;

  if (threadIdx.x == 0) {
    for (int w = 0; w < C::NWG; ++w) {
      PipeCtrl* pc = &ctl->pipe[w];
      for (int s = 0; s < 2; ++s) {
        mbar_init(&pc->bm_full[s], 1);
        mbar_init(&pc->bm_empty[s], 5);  // the 4 softmax warps and the V warp
        mbar_init(&pc->sbar[s], 1);
      }
      mbar_init(&pc->qfull, 32);
      mbar_init(&pc->qempty, 1);
      for (int s = 0; s < C::NKS; ++s) {
        mbar_init(&pc->kfull[s], 32);
        mbar_init(&pc->kempty[s], 1);
      }
      for (int s = 0; s < C::NVS; ++s) {
        mbar_init(&pc->vfull[s], 32);
        mbar_init(&pc->vempty[s], 1);
      }
      mbar_init(&pc->obar, 1);
      mbar_init(&pc->fbar, 1);
    }
    ctl->abort.v = 0;
    fence_mbar_init();
  }
  // P^T buffers start at zero (a stale NaN pattern times a zero V row would
  // still be NaN); for d = 64 the zero tile completes the O^T A operand.
  for (int w = 0; w < C::NWG; ++w) {
    uint4* p = reinterpret_cast<uint4*>(smem + w * C::WG_BYTES + C::OFF_P);
    for (int i = threadIdx.x; i < 2 * C::P_BYTES / 16; i += C::THREADS) p[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  if constexpr (C::PAD_A) {
    uint4* z = reinterpret_cast<uint4*>(smem + C::OFF_PAD);
    for (int i = threadIdx.x; i < C::CHATOM / 16; i += C::THREADS) z[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (wgi == C::COPY_WG) {
    if constexpr (C::NWG > 1) setmaxnreg_dec<C::REGS_COPY>();
    const int cw = warp & 3;  // copy warp: pipeline cw / 2, K (even) or V (odd)
    const int pipe = cw >> 1;
    if (pipe < C::NWG) {
      uint8_t* base = smem + pipe * C::WG_BYTES;
      if ((cw & 1) == 0)
        copy_warp_qk<D>(args, base, &ctl->pipe[pipe], &ctl->abort, pipe);
      else
        copy_warp_v<D>(args, base, &ctl->pipe[pipe], &ctl->abort, pipe);
    }
  } else {
    if constexpr (C::NWG > 1) setmaxnreg_inc<C::REGS_SOFTMAX>();
    softmax_wg<D>(args, smem, ctl, tmem, wgi);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace keys
}  // namespace bsa
