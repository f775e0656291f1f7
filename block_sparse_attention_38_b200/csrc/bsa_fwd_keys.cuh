// bsa_fwd_keys.cuh -- key-tile forward kernel for 32-token blocks.
//
// With 32-token blocks a block row holds only 32 queries, a quarter of the
// 128-row M dimension of a single-CTA tcgen05.mma.  The columns of one block
// row differ from those of its neighbours (log-stride blocks rarely
// coincide), so a tile of four block rows would compute their union, about
// 2.5 times the useful work.  This kernel puts the *keys* on M instead:
//
//   tile  = one block row (b, h, r): 32 queries, its L column blocks;
//   chunk = 4 of those column blocks gathered by TMA into 128 key rows;
//   S^T   = K_chunk Q^T          (M=128 keys, N=32 queries, K=d) -> TMEM;
//   O^T  += V_chunk^T P^T        (M=d rows, N=32 queries, K=128 keys) -> TMEM.
//
// Thread t of a softmax warpgroup owns key row t of a chunk and reads its 32
// query scores with one tcgen05.ld.  The restricted softmax ("Block Sparse
// Attention with Log-Linear Complexity", section 3.3: the denominator sums
// only over the connected key blocks) needs per-query statistics across key
// rows, so they come from a warp transpose-reduction (31 shuffles for 32
// queries) plus a 4-warp exchange in shared memory, once per group of up to
// kChunksResident chunks kept in TMEM: pass 1 takes the exact row maximum,
// pass 2 writes P^T = 2^(s - max) in bf16 and accumulates the fp32 row sums,
// which are transpose-reduced once per tile.  For d = 64 the O^T MMA still
// uses M = 128 (the single-CTA shape whose TMEM layout is one row per lane):
// the upper 64 rows of its A operand are a constant zero tile and rows
// 64..127 of O^T are ignored.  Rows longer than kChunksResident chunks are
// processed in groups with the usual rescaling of O^T and the sums between
// groups.
//
// Warps: 0-3 and 4-7 are two softmax warpgroups working on alternate tiles
// (each with its own TMEM slot of 256 columns), 8 builds the tile's column
// bitmap and streams Q and K, 9 streams V, 10 issues the MMAs.  A missing
// block of a partial chunk is fetched at a row coordinate past the end of the
// tensor, which TMA fills with zeros.
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace keys {

constexpr int kThreads = 352;
constexpr int kChunksResident = 7;        // S^T chunks held in one TMEM slot
constexpr uint32_t kSlotCols = 256;
constexpr uint32_t kOCol = 224;           // O^T columns inside a slot

template <int D>
struct Cfg {
  static constexpr int KATOMS = D / 64;
  static constexpr int Q_BYTES = 32 * D * 2;      // one slot's Q: 32 rows
  static constexpr int QATOM = 32 * 128;          // 32 rows x 128 B
  static constexpr int CH_BYTES = 128 * D * 2;    // one K or V chunk: 128 key rows
  static constexpr int CHATOM = 128 * 128;        // 128 rows x 128 B
  static constexpr int NK = (D == 64) ? 3 : 2;   // K chunk ring
  static constexpr int NV = (D == 64) ? 3 : 2;   // V chunk ring
  static constexpr int NP = 4;                    // P^T buffers per slot
  static constexpr int P_BYTES = 128 * 32 * 2;    // 128 keys x 32 queries, bf16
  static constexpr bool PAD_A = (D == 64);        // zero upper half of the O^T A operand
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * CH_BYTES;
  static constexpr int OFF_PAD = OFF_V + NV * CH_BYTES;
  static constexpr int OFF_P = OFF_PAD + (PAD_A ? CHATOM : 0);
  static constexpr int OFF_CTRL = OFF_P + 2 * NP * P_BYTES;
  static_assert(Q_BYTES % 1024 == 0 && CH_BYTES % 1024 == 0 && P_BYTES % 1024 == 0, "alignment");
};

struct Ctrl {
  uint64_t bm_full[2], bm_empty[2];
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2][4], p_empty[2][4];
  uint64_t pv_done[2], o_free[2];
  uint64_t final_bar;
  uint32_t tmem_base;
  AbortFlag abort;
  uint32_t bitmap[2][kMaxBitmapWords];
  float red[2][4][32];
  float bcast[2][32];
  float lsum[2][32];
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

struct TileInfo {
  long long bh;
  int r, h, L;
};

__device__ __forceinline__ TileInfo tile_info(const FwdArgs& a, long long tile) {
  TileInfo ti;
  ti.bh = tile / a.M;
  ti.r = static_cast<int>(tile - ti.bh * a.M);
  ti.h = static_cast<int>(ti.bh % a.H);
  ti.L = 0;
  return ti;
}

__device__ __forceinline__ int popcount_words(const uint32_t* w, int W) {
  int n = 0;
  for (int i = 0; i < W; ++i) n += __popc(w[i]);
  return n;
}

// ------------------------------------------------------- Q / K producer warp
template <int D>
__device__ void producer_qk(const CUtensorMap* tmQ, const CUtensorMap* tmK, const FwdArgs& a,
                            uint8_t* smem, Ctrl* ctl) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  uint32_t k_loads = 0, q_loads[2] = {0, 0};
  bool ok = true;
  if (lane == 0) {
    prefetch_tensormap(tmQ);
    prefetch_tensormap(tmK);
  }
  int k = 0;
  for (long long tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x, ++k) {
    const int slot = k & 1;
    int w_ok = 1;
    if (lane == 0) w_ok = wait_bounded(&ctl->bm_empty[slot], ((k >> 1) & 1) ^ 1, &ctl->abort);
    if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
    uint32_t* bm = ctl->bitmap[slot];
    for (int w = lane; w < a.W; w += 32) bm[w] = 0u;
    __syncwarp();
    const TileInfo ti = tile_info(a, tile);
    const int beg = __ldg(a.row_ptr + (static_cast<long long>(ti.h) * a.M + ti.r));
    const int end = __ldg(a.row_ptr + (static_cast<long long>(ti.h) * a.M + ti.r + 1));
    if (end < beg) {
      if (lane == 0) atomicOr(&g_status, BSA_STATUS_BAD_ROW_PTR);
    } else {
      for (int p = beg + lane; p < end; p += 32) {
        const int j = __ldg(a.col_idx + p);
        if (j < 0 || j >= a.M) {
          atomicOr(&g_status, BSA_STATUS_BAD_COLUMN);
          continue;
        }
        if (a.causal && j > ti.r) continue;  // wholly above the diagonal: no allowed key
        atomicOr(&bm[j >> 5], 1u << (j & 31));
      }
    }
    __threadfence_block();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&ctl->bm_full[slot]);
      const int L = popcount_words(bm, a.W);
      if (L > 0) {
        ok = wait_bounded(&ctl->q_empty[slot], (q_loads[slot] & 1) ^ 1, &ctl->abort);
        if (ok) {
          mbar_arrive_expect_tx(&ctl->q_full[slot], C::Q_BYTES);
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_load_3d(smem + C::OFF_Q + slot * C::Q_BYTES + ka * C::QATOM, tmQ,
                        &ctl->q_full[slot], ka * 64, ti.r * 32, static_cast<int>(ti.bh));
          ++q_loads[slot];
        }
        BitIter it(bm, a.W);
        const int nch = (L + 3) / 4;
        for (int c = 0; ok && c < nch; ++c) {
          const uint32_t ks = k_loads % C::NK;
          ok = wait_bounded(&ctl->k_empty[ks], ((k_loads / C::NK) & 1) ^ 1, &ctl->abort);
          if (!ok) break;
          mbar_arrive_expect_tx(&ctl->k_full[ks], C::CH_BYTES);
          for (int b = 0; b < 4; ++b) {
            const int j = it.next();
            const int row = j >= 0 ? j * 32 : a.N;  // past the end: zero-filled by TMA
            for (int ka = 0; ka < C::KATOMS; ++ka)
              tma_load_3d(smem + C::OFF_K + ks * C::CH_BYTES + ka * C::CHATOM + b * 4096, tmK,
                          &ctl->k_full[ks], ka * 64, row, static_cast<int>(ti.bh));
          }
          ++k_loads;
        }
      }
    }
    if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { ok = false; break; }
  }
  if (!ok && lane == 0) {
    for (int s = 0; s < 2; ++s)
      if (q_loads[s] > 0) wait_drain(&ctl->q_full[s], (q_loads[s] - 1) & 1);
    for (uint32_t s = 0; s < static_cast<uint32_t>(C::NK); ++s)
      if (k_loads > s) {
        const uint32_t last = s + C::NK * ((k_loads - 1 - s) / C::NK);
        wait_drain(&ctl->k_full[s], (last / C::NK) & 1);
      }
  }
  __syncwarp();
}

// --------------------------------------------------------------- V producer
template <int D>
__device__ void producer_v(const CUtensorMap* tmV, const FwdArgs& a, uint8_t* smem, Ctrl* ctl) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  uint32_t v_loads = 0;
  bool ok = true;
  if (lane == 0) {
    prefetch_tensormap(tmV);
    int k = 0;
    for (long long tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x, ++k) {
      const int slot = k & 1;
      if (!wait_bounded(&ctl->bm_full[slot], (k >> 1) & 1, &ctl->abort)) { ok = false; break; }
      const TileInfo ti = tile_info(a, tile);
      const uint32_t* bm = ctl->bitmap[slot];
      const int L = popcount_words(bm, a.W);
      BitIter it(bm, a.W);
      const int nch = (L + 3) / 4;
      for (int c = 0; c < nch; ++c) {
        const uint32_t vs = v_loads % C::NV;
        ok = wait_bounded(&ctl->v_empty[vs], ((v_loads / C::NV) & 1) ^ 1, &ctl->abort);
        if (!ok) break;
        mbar_arrive_expect_tx(&ctl->v_full[vs], C::CH_BYTES);
        for (int b = 0; b < 4; ++b) {
          const int j = it.next();
          const int row = j >= 0 ? j * 32 : a.N;
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_load_3d(smem + C::OFF_V + vs * C::CH_BYTES + ka * C::CHATOM + b * 4096, tmV,
                        &ctl->v_full[vs], ka * 64, row, static_cast<int>(ti.bh));
        }
        ++v_loads;
      }
      mbar_arrive(&ctl->bm_empty[slot]);
    }
    if (!ok)
      for (uint32_t s = 0; s < static_cast<uint32_t>(C::NV); ++s)
        if (v_loads > s) {
          const uint32_t last = s + C::NV * ((v_loads - 1 - s) / C::NV);
          wait_drain(&ctl->v_full[s], (last / C::NV) & 1);
        }
  }
  __syncwarp();
}

// ------------------------------------------------------------------ MMA warp
struct Item {
  int k;        // CTA-local tile index
  int slot;
  int c0, nc;   // first chunk of the group and its chunk count
  bool first, last;
};

template <int D>
struct MmaState {
  uint32_t k_cons = 0, v_cons = 0;
  uint32_t q_uses[2] = {0, 0}, s_uses[2] = {0, 0}, chunks[2] = {0, 0}, o_uses[2] = {0, 0};
};

template <int D>
__device__ bool issue_qk(const Item& X, MmaState<D>& st, uint8_t* smem, Ctrl* ctl, uint32_t tmem) {
  using C = Cfg<D>;
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, 32, false, false);
  const int s = X.slot;
  if (X.first) {
    if (!wait_bounded(&ctl->q_full[s], st.q_uses[s] & 1, &ctl->abort)) return false;
    ++st.q_uses[s];
  }
  if (!wait_bounded(&ctl->s_free[s], (st.s_uses[s] & 1) ^ 1, &ctl->abort)) return false;
  ++st.s_uses[s];
  const uint32_t q_base = smem_u32(smem + C::OFF_Q + s * C::Q_BYTES);
  const uint32_t k_base = smem_u32(smem + C::OFF_K);
  for (int c = 0; c < X.nc; ++c) {
    const uint32_t ks = st.k_cons % C::NK;
    if (!wait_bounded(&ctl->k_full[ks], (st.k_cons / C::NK) & 1, &ctl->abort)) return false;
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t ad = sdesc_sw128(k_base + ks * C::CH_BYTES + (kk >> 2) * C::CHATOM + (kk & 3) * 32,
                                      16, 1024);
      const uint64_t bd = sdesc_sw128(q_base + (kk >> 2) * C::QATOM + (kk & 3) * 32, 16, 1024);
      umma_bf16_ss(tmem + s * kSlotCols + c * 32, ad, bd, kIdesc, kk > 0 ? 1u : 0u);
    }
    umma_commit(&ctl->k_empty[ks]);
    ++st.k_cons;
  }
  umma_commit(&ctl->s_full[s]);
  if (X.last) umma_commit(&ctl->q_empty[s]);
  return true;
}

template <int D>
__device__ bool issue_pv(const Item& X, MmaState<D>& st, uint8_t* smem, Ctrl* ctl, uint32_t tmem) {
  using C = Cfg<D>;
  // A = V^T (MN-major, 128-byte swizzle), B = P^T (MN-major, 64-byte swizzle).
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, 32, true, true);
  const int s = X.slot;
  if (X.first) {
    if (!wait_bounded(&ctl->o_free[s], (st.o_uses[s] & 1) ^ 1, &ctl->abort)) return false;
    ++st.o_uses[s];
  }
  const uint32_t v_base = smem_u32(smem + C::OFF_V);
  const uint32_t pad = smem_u32(smem + C::OFF_PAD);
  const uint32_t p_base = smem_u32(smem + C::OFF_P + s * C::NP * C::P_BYTES);
  for (int c = 0; c < X.nc; ++c) {
    const uint32_t g = st.chunks[s];
    const uint32_t pb = g % C::NP;
    if (!wait_bounded(&ctl->p_full[s][pb], (g / C::NP) & 1, &ctl->abort)) return false;
    const uint32_t vs = st.v_cons % C::NV;
    if (!wait_bounded(&ctl->v_full[vs], (st.v_cons / C::NV) & 1, &ctl->abort)) return false;
    tc_fence_after();
    const uint32_t vstage = v_base + vs * C::CH_BYTES;
    const uint32_t lbo = C::PAD_A ? (pad - vstage) : static_cast<uint32_t>(C::CHATOM);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {  // 128 keys, 16 per MMA
      const uint64_t ad = sdesc(vstage + kk * 2048, lbo, 1024, kLayoutSW128);
      const uint64_t bd = sdesc(p_base + pb * C::P_BYTES + kk * 1024, C::P_BYTES, 512, kLayoutSW64);
      umma_bf16_ss(tmem + s * kSlotCols + kOCol, ad, bd, kIdesc,
                   (X.first && c == 0 && kk == 0) ? 0u : 1u);
    }
    umma_commit(&ctl->v_empty[vs]);
    umma_commit(&ctl->p_empty[s][pb]);
    ++st.v_cons;
    ++st.chunks[s];
  }
  umma_commit(&ctl->pv_done[s]);
  return true;
}

template <int D>
__device__ void mma_role(const FwdArgs& a, uint8_t* smem, Ctrl* ctl, uint32_t tmem) {
  MmaState<D> st;
  Item pending{};
  bool has_pending = false;
  bool ok = true;
  int k = 0;
  for (long long tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x, ++k) {
    const int slot = k & 1;
    if (!wait_bounded(&ctl->bm_full[slot], (k >> 1) & 1, &ctl->abort)) { ok = false; break; }
    const int L = popcount_words(ctl->bitmap[slot], a.W);
    mbar_arrive(&ctl->bm_empty[slot]);
    if (L == 0) continue;
    const int nch = (L + 3) / 4;
    for (int c0 = 0; ok && c0 < nch; c0 += kChunksResident) {
      Item X;
      X.k = k;
      X.slot = slot;
      X.c0 = c0;
      X.nc = min(kChunksResident, nch - c0);
      X.first = (c0 == 0);
      X.last = (c0 + kChunksResident >= nch);
      // QK of a new tile goes ahead of the PV of the previous tile, so one
      // warpgroup's softmax overlaps the other's tensor-core work; within a
      // tile the next group's QK waits for this group's PV.
      if (has_pending && pending.k == k) {
        ok = issue_pv<D>(pending, st, smem, ctl, tmem) && issue_qk<D>(X, st, smem, ctl, tmem);
      } else {
        ok = issue_qk<D>(X, st, smem, ctl, tmem);
        if (ok && has_pending) ok = issue_pv<D>(pending, st, smem, ctl, tmem);
      }
      pending = X;
      has_pending = true;
    }
  }
  if (ok && has_pending) issue_pv<D>(pending, st, smem, ctl, tmem);
  umma_commit(&ctl->final_bar);
  wait_drain(&ctl->final_bar, 0);
}

// --------------------------------------------------------- softmax warpgroups
template <int D>
__device__ void softmax_role(const FwdArgs& a, uint8_t* smem, Ctrl* ctl, uint32_t tmem, int wg) {
  using C = Cfg<D>;
  const int tid = threadIdx.x & 127;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int slot = wg;
  const uint32_t t_lane = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t s_col = tmem + slot * kSlotCols + t_lane;
  const uint32_t o_col = tmem + slot * kSlotCols + kOCol + t_lane;
  const uint32_t p_row0 = smem_u32(smem + C::OFF_P + slot * C::NP * C::P_BYTES) + tid * 64;
  const int bar_id = 1 + slot;
  constexpr float kNegInf = -INFINITY;
  uint32_t s_uses = 0, chunks = 0, pv_waits = 0;

  for (int k = wg;; k += 2) {
    const long long tile = blockIdx.x + static_cast<long long>(k) * gridDim.x;
    if (tile >= a.num_tiles) break;
    if (!warp_wait(&ctl->bm_full[slot], (k >> 1) & 1, &ctl->abort)) return;
    const uint32_t* bm = ctl->bitmap[slot];
    const TileInfo ti = tile_info(a, tile);
    const int L = popcount_words(bm, a.W);
    int diag_pos = -1;
    if (a.causal && ((bm[ti.r >> 5] >> (ti.r & 31)) & 1u)) {
      diag_pos = 0;
      for (int w = 0; w < (ti.r >> 5); ++w) diag_pos += __popc(bm[w]);
      diag_pos += __popc(bm[ti.r >> 5] & ((1u << (ti.r & 31)) - 1u));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->bm_empty[slot]);
    const long long row0 = ti.bh * a.N + static_cast<long long>(ti.r) * 32;  // first query row

    if (L == 0) {  // no key at all: O = 0, LSE = -inf
      uint4* o = reinterpret_cast<uint4*>(a.O + row0 * D);
      for (int i = tid; i < 32 * D / 8; i += 128) o[i] = make_uint4(0u, 0u, 0u, 0u);
      if (warp == 0) a.LSE[row0 + lane] = kNegInf;
      continue;
    }

    const int nch = (L + 3) / 4;
    float mu[32];     // running max per query (log2 units), -inf replaced by 0
    float lpart[32];  // this thread's partial row sums
    float m_own = kNegInf;  // running max of query `lane`, -inf kept
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      mu[q] = 0.f;
      lpart[q] = 0.f;
    }
    for (int c0 = 0; c0 < nch; c0 += kChunksResident) {
      const int nc = min(kChunksResident, nch - c0);
      if (!warp_wait(&ctl->s_full[slot], s_uses & 1, &ctl->abort)) return;
      ++s_uses;
      tc_fence_after();

      // ---- pass 1: per-query maximum over the key rows of this group
      float mx[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) mx[q] = kNegInf;
      for (int c = 0; c < nc; ++c) {
        const int blk = 4 * (c0 + c) + warp;  // block slot held by this warp
        if (blk < L) {
          uint32_t u[32];
          tmem_ld32(s_col + c * 32, u);
          tmem_wait_ld();
          if (blk == diag_pos) {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const float v = (lane > q) ? kNegInf : __uint_as_float(u[q]) * a.scale_log2;
              mx[q] = fmaxf(mx[q], v);
            }
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) mx[q] = fmaxf(mx[q], __uint_as_float(u[q]) * a.scale_log2);
          }
        }
      }
      const float wmax = transpose_reduce(mx, [](float x, float y) { return fmaxf(x, y); });
      ctl->red[slot][warp][lane] = wmax;
      named_bar(bar_id, 128);
      const float gmax = fmaxf(fmaxf(ctl->red[slot][0][lane], ctl->red[slot][1][lane]),
                               fmaxf(ctl->red[slot][2][lane], ctl->red[slot][3][lane]));
      const float m_new_own = fmaxf(m_own, gmax);
      if (warp == 0) ctl->bcast[slot][lane] = (m_new_own == kNegInf) ? 0.f : m_new_own;
      named_bar(bar_id, 128);
      m_own = m_new_own;
      float mnew[32];
#pragma unroll
      for (int q = 0; q < 32; q += 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(&ctl->bcast[slot][q]);
        mnew[q] = t4.x;
        mnew[q + 1] = t4.y;
        mnew[q + 2] = t4.z;
        mnew[q + 3] = t4.w;
      }

      // ---- rescale what earlier groups of this row accumulated
      if (c0 > 0) {
        if (!warp_wait(&ctl->pv_done[slot], pv_waits & 1, &ctl->abort)) return;
        ++pv_waits;
        tc_fence_after();
        uint32_t u[32];
        tmem_ld32(o_col, u);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const float f = ex2_approx(mu[q] - mnew[q]);
          u[q] = __float_as_uint(__uint_as_float(u[q]) * f);
          lpart[q] *= f;
        }
        tmem_st32(o_col, u);
        tmem_wait_st();
      }
#pragma unroll
      for (int q = 0; q < 32; ++q) mu[q] = mnew[q];

      // ---- pass 2: P^T = 2^(s - max) in bf16, chunk by chunk
      for (int c = 0; c < nc; ++c) {
        const uint32_t pb = chunks % C::NP;
        if (!warp_wait(&ctl->p_empty[slot][pb], ((chunks / C::NP) & 1) ^ 1, &ctl->abort)) return;
        const int blk = 4 * (c0 + c) + warp;
        if (blk < L) {
          uint32_t u[32];
          tmem_ld32(s_col + c * 32, u);
          tmem_wait_ld();
          const bool diag = (blk == diag_pos);
          uint32_t pk[16];
#pragma unroll
          for (int q = 0; q < 32; q += 2) {
            float x0 = __uint_as_float(u[q]) * a.scale_log2 - mu[q];
            float x1 = __uint_as_float(u[q + 1]) * a.scale_log2 - mu[q + 1];
            if (diag && lane > q) x0 = kNegInf;
            if (diag && lane > q + 1) x1 = kNegInf;
            const float p0 = ex2_approx(x0);
            const float p1 = ex2_approx(x1);
            lpart[q] += p0;
            lpart[q + 1] += p1;
            pk[q >> 1] = pack_bf16x2(p0, p1);
          }
          // row `tid` of P^T (64 bytes), 64-byte swizzle: chunk c sits at c ^ ((tid >> 1) & 3)
          const uint32_t base = p_row0 + pb * C::P_BYTES;
          const uint32_t sw = (tid >> 1) & 3;
#pragma unroll
          for (int c16 = 0; c16 < 4; ++c16)
            st_shared_v4(base + ((c16 ^ sw) << 4), pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2],
                         pk[4 * c16 + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->p_full[slot][pb]);
        ++chunks;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->s_free[slot]);
    }

    // ---- epilogue: O = O^T / l, LSE = (max + log2 l) ln 2
    if (!warp_wait(&ctl->pv_done[slot], pv_waits & 1, &ctl->abort)) return;
    ++pv_waits;
    tc_fence_after();
    uint32_t u[32];
    tmem_ld32(o_col, u);
    tmem_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->o_free[slot]);
    {
      const float wsum = transpose_reduce(lpart, [](float x, float y) { return x + y; });
      ctl->red[slot][warp][lane] = wsum;
      named_bar(bar_id, 128);
      if (warp == 0)
        ctl->lsum[slot][lane] = (ctl->red[slot][0][lane] + ctl->red[slot][1][lane]) +
                                (ctl->red[slot][2][lane] + ctl->red[slot][3][lane]);
    }
    named_bar(bar_id, 128);
    if (warp < D / 32) {
      const int d = tid;  // O^T row = head-dim index
      __nv_bfloat16* orow = a.O + row0 * D + d;
#pragma unroll
      for (int q = 0; q < 32; q += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(&ctl->lsum[slot][q]);
        const float ls[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float inv = ls[i] > 0.f ? 1.f / ls[i] : 0.f;
          orow[static_cast<long long>(q + i) * D] = __float2bfloat16_rn(__uint_as_float(u[q + i]) * inv);
        }
      }
    }
    if (warp == 3) {
      const float l = ctl->lsum[slot][lane];
      a.LSE[row0 + lane] = l > 0.f ? (m_own + __log2f(l)) * 0.69314718055994531f : kNegInf;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdArgs args) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Ctrl* ctl = reinterpret_cast<Ctrl*>(smem + C::OFF_CTRL);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->bm_full[s], 1);
      mbar_init(&ctl->bm_empty[s], 6);  // softmax warps of the slot (4) + MMA + V producer
      mbar_init(&ctl->q_full[s], 1);
      mbar_init(&ctl->q_empty[s], 1);
      mbar_init(&ctl->s_full[s], 1);
      mbar_init(&ctl->s_free[s], 4);
      mbar_init(&ctl->pv_done[s], 1);
      mbar_init(&ctl->o_free[s], 4);
      for (int b = 0; b < 4; ++b) {
        mbar_init(&ctl->p_full[s][b], 4);
        mbar_init(&ctl->p_empty[s][b], 1);
      }
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->k_empty[s], 1);
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->v_empty[s], 1);
    }
    mbar_init(&ctl->final_bar, 1);
    ctl->abort.v = 0;
    fence_mbar_init();
  }
  if (warp < 8) {
    // P^T buffers start at zero (a stale NaN pattern times a zero V row would
    // still be NaN); for d = 64 the zero tile completes the O^T A operand.
    uint4* p = reinterpret_cast<uint4*>(smem + C::OFF_P);
    for (int i = threadIdx.x; i < 2 * C::NP * C::P_BYTES / 16; i += 256) p[i] = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (C::PAD_A) {
      uint4* z = reinterpret_cast<uint4*>(smem + C::OFF_PAD);
      for (int i = threadIdx.x; i < C::CHATOM / 16; i += 256) z[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  if (warp == 10) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp < 8) {
    softmax_role<D>(args, smem, ctl, tmem, warp >> 2);
    __syncwarp();
  } else if (warp == 8) {
    producer_qk<D>(&tmQ, &tmK, args, smem, ctl);
  } else if (warp == 9) {
    producer_v<D>(&tmV, args, smem, ctl);
  } else {
    if ((threadIdx.x & 31) == 0) mma_role<D>(args, smem, ctl, tmem);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 10) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace keys
}  // namespace bsa
