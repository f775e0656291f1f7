// bsa_fwd_rows.cuh -- row-tile forward kernel (block_size 64 and 128).
//
// A tile is 128 query rows = 128 / block_size consecutive block rows of one
// (b, h).  Q rows sit on the MMA's M dimension; for every column j of the
// union of the tile's block rows the kernel computes S = Q K_j^T (M=128,
// N=block_size) into TMEM, runs the restricted online softmax with one thread
// per query row, and accumulates O += P V_j (M=128, N=d) into TMEM.  A block
// row that does not hold column j gets P = 0 for it and keeps its statistics,
// so every row sums exactly over its own blocks ("Block Sparse Attention with
// Log-Linear Complexity", section 3.3).
//
// Warp roles (one persistent CTA per SM): warp 4 = TMA producer and bitmap
// builder, warp 5 = tcgen05.mma issuer, warps 0-3 = softmax / correction /
// epilogue.
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace rows {

constexpr int kThreads = 192;

template <int BS, int D>
struct Cfg {
  static constexpr int TM = 128;                 // query rows per tile
  static constexpr int R = TM / BS;              // block rows per tile
  static constexpr int KATOMS = D / 64;          // 128-byte column atoms of a D-wide row
  static constexpr int Q_BYTES = TM * D * 2;
  static constexpr int KV_BYTES = BS * D * 2;    // one K or one V block
  static constexpr int P_ATOMS = (BS + 63) / 64;
  static constexpr int P_BYTES = P_ATOMS * TM * 128;
  static constexpr int BUDGET = 200 * 1024;
  static constexpr int ST_FIT = (BUDGET - Q_BYTES - P_BYTES) / (2 * KV_BYTES);
  static constexpr int STAGES = ST_FIT > 4 ? 4 : ST_FIT;
  static_assert(STAGES >= 2, "not enough shared memory for a double-buffered K/V ring");
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = OFF_Q + Q_BYTES;
  static constexpr int OFF_K = OFF_P + P_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_CTRL = OFF_V + STAGES * KV_BYTES;
  static constexpr uint32_t TMEM_S = 0;          // two score buffers of BS fp32 columns
  static constexpr uint32_t TMEM_O = 256;        // O accumulator, D fp32 columns
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(2 * BS <= 256 && D <= 256, "TMEM layout");
  static_assert((Q_BYTES % 1024) == 0 && (KV_BYTES % 1024) == 0 && (P_BYTES % 1024) == 0,
                "1024-byte alignment of swizzled tiles");
};

struct Ctrl {
  uint64_t q_full, q_empty;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, pv_done, o_empty;
  uint64_t bm_full[2], bm_empty[2];
  uint64_t final_bar;
  uint32_t tmem_base;
  AbortFlag abort;
  uint32_t bitmap[2][5 * kMaxBitmapWords];  // per tile: R block-row maps, then their union
};

// ------------------------------------------------------------- producer warp
template <int BS, int D>
__device__ void producer_role(const CUtensorMap* tmQ, const CUtensorMap* tmK,
                              const CUtensorMap* tmV, const FwdArgs& a, uint8_t* smem, Ctrl* ctl) {
  using C = Cfg<BS, D>;
  const int lane = threadIdx.x & 31;
  uint32_t q_loads = 0, k_loads = 0, v_loads = 0;
  bool ok = true;
  if (lane == 0) {
    prefetch_tensormap(tmQ);
    prefetch_tensormap(tmK);
    prefetch_tensormap(tmV);
  }
  int t = 0;
  for (long long tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x, ++t) {
    const int buf = t & 1;
    int w_ok = 1;
    if (lane == 0) w_ok = wait_bounded(&ctl->bm_empty[buf], ((t >> 1) & 1) ^ 1, &ctl->abort);
    if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }

    uint32_t* bm = ctl->bitmap[buf];
    const int W = a.W;
    for (int w = lane; w < (C::R + 1) * W; w += 32) bm[w] = 0u;
    __syncwarp();
    const long long bh = tile / a.G;
    const int g = static_cast<int>(tile - bh * a.G);
    const int h = static_cast<int>(bh % a.H);
    for (int i = 0; i < C::R; ++i) {
      const int r = g * C::R + i;
      if (r >= a.M) break;
      const int beg = __ldg(a.row_ptr + (static_cast<long long>(h) * a.M + r));
      const int end = __ldg(a.row_ptr + (static_cast<long long>(h) * a.M + r + 1));
      if (end < beg) {
        if (lane == 0) atomicOr(&g_status, BSA_STATUS_BAD_ROW_PTR);
        continue;
      }
      for (int p = beg + lane; p < end; p += 32) {
        const int j = __ldg(a.col_idx + p);
        if (j < 0 || j >= a.M) {
          atomicOr(&g_status, BSA_STATUS_BAD_COLUMN);
          continue;
        }
        if (a.causal && j > r) continue;  // a block wholly above the diagonal has no allowed key
        atomicOr(&bm[i * W + (j >> 5)], 1u << (j & 31));
        atomicOr(&bm[C::R * W + (j >> 5)], 1u << (j & 31));
      }
    }
    __threadfence_block();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&ctl->bm_full[buf]);
      const uint32_t* uni = bm + C::R * W;
      const int n = union_count(uni, W);
      if (n > 0) {
        ok = wait_bounded(&ctl->q_empty, (q_loads & 1) ^ 1, &ctl->abort);
        if (ok) {
          mbar_arrive_expect_tx(&ctl->q_full, C::Q_BYTES);
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_load_3d(smem + C::OFF_Q + ka * (C::TM * 128), tmQ, &ctl->q_full, ka * 64,
                        g * C::TM, static_cast<int>(bh));
          ++q_loads;
        }
        BitIter it(uni, W);
        for (int j = it.next(); ok && j >= 0; j = it.next()) {
          const uint32_t ks = k_loads % C::STAGES;
          ok = wait_bounded(&ctl->k_empty[ks], ((k_loads / C::STAGES) & 1) ^ 1, &ctl->abort);
          if (!ok) break;
          mbar_arrive_expect_tx(&ctl->k_full[ks], C::KV_BYTES);
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_load_3d(smem + C::OFF_K + ks * C::KV_BYTES + ka * (BS * 128), tmK,
                        &ctl->k_full[ks], ka * 64, j * BS, static_cast<int>(bh));
          ++k_loads;
          const uint32_t vs = v_loads % C::STAGES;
          ok = wait_bounded(&ctl->v_empty[vs], ((v_loads / C::STAGES) & 1) ^ 1, &ctl->abort);
          if (!ok) break;
          mbar_arrive_expect_tx(&ctl->v_full[vs], C::KV_BYTES);
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_load_3d(smem + C::OFF_V + vs * C::KV_BYTES + ka * (BS * 128), tmV,
                        &ctl->v_full[vs], ka * 64, j * BS, static_cast<int>(bh));
          ++v_loads;
        }
      }
    }
    if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { ok = false; break; }
  }
  // On an early exit, let every copy already issued land before the CTA ends.
  if (!ok && lane == 0) {
    if (q_loads > 0) wait_drain(&ctl->q_full, (q_loads - 1) & 1);
    for (uint32_t s = 0; s < C::STAGES; ++s) {
      if (k_loads > s) {
        const uint32_t last = s + C::STAGES * ((k_loads - 1 - s) / C::STAGES);
        wait_drain(&ctl->k_full[s], (last / C::STAGES) & 1);
      }
      if (v_loads > s) {
        const uint32_t last = s + C::STAGES * ((v_loads - 1 - s) / C::STAGES);
        wait_drain(&ctl->v_full[s], (last / C::STAGES) & 1);
      }
    }
  }
  __syncwarp();
}

// ------------------------------------------------------------------ MMA warp
template <int BS, int D>
__device__ void mma_role(const FwdArgs& a, uint8_t* smem, Ctrl* ctl, uint32_t tmem) {
  using C = Cfg<BS, D>;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, BS, false, false);  // Q, K both K-major
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);    // P K-major, V MN-major
  const uint32_t q_base = smem_u32(smem + C::OFF_Q);
  const uint32_t p_base = smem_u32(smem + C::OFF_P);
  const uint32_t k_base = smem_u32(smem + C::OFF_K);
  const uint32_t v_base = smem_u32(smem + C::OFF_V);
  uint32_t k_cons = 0, v_cons = 0, s_iter = 0, pv_iter = 0, q_uses = 0, nonempty = 0;
  bool ok = true;

  // S[sb] = Q K^T for the next K block in the ring.
  auto issue_qk = [&](bool last_of_tile) -> bool {
    const uint32_t sb = s_iter & 1;
    if (!wait_bounded(&ctl->s_empty[sb], ((s_iter >> 1) & 1) ^ 1, &ctl->abort)) return false;
    const uint32_t ks = k_cons % C::STAGES;
    if (!wait_bounded(&ctl->k_full[ks], (k_cons / C::STAGES) & 1, &ctl->abort)) return false;
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t ad =
          sdesc_sw128(q_base + (kk >> 2) * (C::TM * 128) + (kk & 3) * 32, 16, 1024);
      const uint64_t bd = sdesc_sw128(
          k_base + ks * C::KV_BYTES + (kk >> 2) * (BS * 128) + (kk & 3) * 32, 16, 1024);
      umma_bf16_ss(tmem + C::TMEM_S + sb * BS, ad, bd, kIdescQK, kk > 0 ? 1u : 0u);
    }
    umma_commit(&ctl->k_empty[ks]);
    umma_commit(&ctl->s_full[sb]);
    if (last_of_tile) umma_commit(&ctl->q_empty);
    ++k_cons;
    ++s_iter;
    return true;
  };

  int t = 0;
  for (long long tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x, ++t) {
    const int buf = t & 1;
    if (!wait_bounded(&ctl->bm_full[buf], (t >> 1) & 1, &ctl->abort)) { ok = false; break; }
    const int n = union_count(ctl->bitmap[buf] + C::R * a.W, a.W);
    if (n > 0) {
      if (!wait_bounded(&ctl->q_full, q_uses & 1, &ctl->abort)) { ok = false; break; }
      ++q_uses;
      tc_fence_after();
      if (!issue_qk(n == 1)) { ok = false; break; }
      for (int e = 0; e < n; ++e) {
        if (e + 1 < n && !issue_qk(e + 2 == n)) { ok = false; break; }
        if (e == 0 && nonempty > 0 &&
            !wait_bounded(&ctl->o_empty, (nonempty - 1) & 1, &ctl->abort)) { ok = false; break; }
        if (!wait_bounded(&ctl->p_full, pv_iter & 1, &ctl->abort)) { ok = false; break; }
        const uint32_t vs = v_cons % C::STAGES;
        if (!wait_bounded(&ctl->v_full[vs], (v_cons / C::STAGES) & 1, &ctl->abort)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BS / 16; ++kk) {
          const uint64_t ad =
              sdesc_sw128(p_base + (kk >> 2) * (C::TM * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t bd =
              sdesc_sw128(v_base + vs * C::KV_BYTES + kk * (16 * 128), BS * 128, 1024);
          umma_bf16_ss(tmem + C::TMEM_O, ad, bd, kIdescPV, (e > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&ctl->v_empty[vs]);
        umma_commit(&ctl->pv_done);
        ++v_cons;
        ++pv_iter;
      }
      if (!ok) break;
      ++nonempty;
    }
    mbar_arrive(&ctl->bm_empty[buf]);
  }
  // Every MMA issued must complete before the TMEM is released.
  umma_commit(&ctl->final_bar);
  wait_drain(&ctl->final_bar, 0);
}

// ------------------------------------------------------------ softmax warps
template <int BS, int D>
__device__ void softmax_role(const FwdArgs& a, uint8_t* smem, Ctrl* ctl, uint32_t tmem) {
  using C = Cfg<BS, D>;
  const int row = threadIdx.x;          // 0..127: query row of the tile
  const int warp = row >> 5;
  const int lane = row & 31;
  const int sub = row / BS;             // block row of the tile this thread belongs to
  const int qq = row % BS;              // position inside that block row
  const uint32_t t_lane = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t p_row = smem_u32(smem + C::OFF_P) + row * 128;
  constexpr float kNegInf = -INFINITY;
  uint32_t s_iter = 0, pv_seen = 0;
  bool p_zero = false;                  // this warp's P rows already hold zeros

  int t = 0;
  for (long long tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x, ++t) {
    const int buf = t & 1;
    if (!warp_wait(&ctl->bm_full[buf], (t >> 1) & 1, &ctl->abort)) return;
    const uint32_t* bm_sub = ctl->bitmap[buf] + sub * a.W;
    const uint32_t* uni = ctl->bitmap[buf] + C::R * a.W;
    const long long bh = tile / a.G;
    const int g = static_cast<int>(tile - bh * a.G);
    const int r_sub = g * C::R + sub;
    const bool row_ok = r_sub < a.M;
    const int n = union_count(uni, a.W);

    float m_used = kNegInf;  // running max in log2 units of the scaled score
    float l = 0.f;           // running sum of 2^(s - m_used)
    BitIter it(uni, a.W);
    for (int e = 0; e < n; ++e) {
      const int j = it.next();
      const bool member = row_ok && ((bm_sub[j >> 5] >> (j & 31)) & 1u);  // warp-uniform
      const uint32_t sb = s_iter & 1;
      if (!warp_wait(&ctl->s_full[sb], (s_iter >> 1) & 1, &ctl->abort)) return;
      tc_fence_after();
      float s[BS];
      if (member) {
#pragma unroll
        for (int c = 0; c < BS / 32; ++c) {
          uint32_t u[32];
          tmem_ld32(tmem + t_lane + C::TMEM_S + sb * BS + c * 32, u);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(u[i]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->s_empty[sb]);
      ++s_iter;

      bool need_rescale = false;
      float factor = 1.f;
      if (member) {
        const bool diag = a.causal && (j == r_sub);
        float mx = kNegInf;
#pragma unroll
        for (int c = 0; c < BS; ++c) {
          float v = s[c] * a.scale_log2;
          if (diag && c > qq) v = kNegInf;  // key after the query (diagonal block only)
          s[c] = v;
          mx = fmaxf(mx, v);
        }
        const float m_new = fmaxf(m_used, mx);
        if (m_new > m_used + kRescaleThreshold) {
          if (l > 0.f) {
            need_rescale = true;
            factor = ex2_approx(m_used - m_new);
          }
          m_used = m_new;
        }
        const float mu = (m_used == kNegInf) ? 0.f : m_used;
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < BS; ++c) {
          const float p = ex2_approx(s[c] - mu);
          s[c] = p;
          rs += p;
        }
        l = l * factor + rs;
      }

      // PV of the previous block must be done before O is rescaled or P overwritten.
      if (e > 0) {
        if (!warp_wait(&ctl->pv_done, pv_seen & 1, &ctl->abort)) return;
        ++pv_seen;
      }
      tc_fence_after();
      if (__any_sync(0xffffffffu, need_rescale)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t u[32];
          tmem_ld32(tmem + t_lane + C::TMEM_O + c * 32, u);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * factor);
          tmem_st32(tmem + t_lane + C::TMEM_O + c * 32, u);
        }
        tmem_wait_st();
      }
      if (member) {
#pragma unroll
        for (int cc = 0; cc < BS / 8; ++cc) {  // 16-byte chunks of 8 keys, 128-byte swizzle
          const uint32_t addr = p_row + (cc >> 3) * (C::TM * 128) + (((cc & 7) ^ (row & 7)) << 4);
          st_shared_v4(addr, pack_bf16x2(s[cc * 8 + 0], s[cc * 8 + 1]),
                       pack_bf16x2(s[cc * 8 + 2], s[cc * 8 + 3]),
                       pack_bf16x2(s[cc * 8 + 4], s[cc * 8 + 5]),
                       pack_bf16x2(s[cc * 8 + 6], s[cc * 8 + 7]));
        }
        p_zero = false;
      } else if (!p_zero) {
#pragma unroll
        for (int cc = 0; cc < BS / 8; ++cc) {
          const uint32_t addr = p_row + (cc >> 3) * (C::TM * 128) + (((cc & 7) ^ (row & 7)) << 4);
          st_shared_v4(addr, 0u, 0u, 0u, 0u);
        }
        p_zero = true;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->p_full);
    }

    // Epilogue: O / l in bf16 and LSE = (m + log2 l) ln 2.
    const long long qtok = static_cast<long long>(g) * C::TM + row;
    __nv_bfloat16* orow = a.O + (bh * a.N + qtok) * D;
    if (n > 0) {
      if (!warp_wait(&ctl->pv_done, pv_seen & 1, &ctl->abort)) return;
      ++pv_seen;
      tc_fence_after();
      float o[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(tmem + t_lane + C::TMEM_O + c * 32, u);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[c * 32 + i] = __uint_as_float(u[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->o_empty);
      if (row_ok) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          uint4 v;
          v.x = pack_bf16x2(o[c * 8 + 0] * inv, o[c * 8 + 1] * inv);
          v.y = pack_bf16x2(o[c * 8 + 2] * inv, o[c * 8 + 3] * inv);
          v.z = pack_bf16x2(o[c * 8 + 4] * inv, o[c * 8 + 5] * inv);
          v.w = pack_bf16x2(o[c * 8 + 6] * inv, o[c * 8 + 7] * inv);
          dst[c] = v;
        }
        a.LSE[bh * a.N + qtok] = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f : kNegInf;
      }
    } else if (row_ok) {
      uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
      a.LSE[bh * a.N + qtok] = kNegInf;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->bm_empty[buf]);
  }
}

template <int BS, int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdArgs args) {
  using C = Cfg<BS, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Ctrl* ctl = reinterpret_cast<Ctrl*>(smem + C::OFF_CTRL);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_empty, 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->k_empty[s], 1);
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->s_full[s], 1);
      mbar_init(&ctl->s_empty[s], 4);
      mbar_init(&ctl->bm_full[s], 1);
      mbar_init(&ctl->bm_empty[s], 5);
    }
    mbar_init(&ctl->p_full, 4);
    mbar_init(&ctl->pv_done, 1);
    mbar_init(&ctl->o_empty, 4);
    mbar_init(&ctl->final_bar, 1);
    ctl->abort.v = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 4) {
    producer_role<BS, D>(&tmQ, &tmK, &tmV, args, smem, ctl);
  } else if (warp == 5) {
    if ((threadIdx.x & 31) == 0) mma_role<BS, D>(args, smem, ctl, tmem);
    __syncwarp();
  } else {
    softmax_role<BS, D>(args, smem, ctl, tmem);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace rows
}  // namespace bsa
