// bsa_fwd_rows.cuh -- row-tile forward kernel (every block size).
//
// A tile is 128 query rows = R = 128 / block_size consecutive block rows of
// one (b, h).  The kernel walks the union of the tile's column lists in steps
// of 128 keys (128 / block_size blocks gathered into one shared-memory stage):
//
//   S = Q K_step^T            tcgen05.mma, M=128 queries, N=128 keys, K=d
//   P = 2^(S*scale*log2e - m) one thread per query row, fp32, written back to
//                             TMEM as bf16 over the first half of S
//   O += P V_step             tcgen05.mma with A = P read from TMEM, N=d
//
// A block row that does not hold a block of the step gets P = 0 there and its
// statistics skip it, so every row sums exactly over its own blocks ("Block
// Sparse Attention with Log-Linear Complexity", section 3.3); the exponentials
// of such blocks are not evaluated (membership is uniform over a warp).
//
// One persistent CTA per SM runs two independent tile slots so that the
// tensor core works on one slot while the other slot's softmax runs.  Roles:
//   warps 0-3   softmax / epilogue of slot 0    warps 4-7  same, slot 1
//   warp 8 + s  bitmap builder + TMA producer of slot s
//   warp 10 + s tcgen05.mma issuer of slot s (warp 10 also owns the TMEM)
// TMEM: slot s uses columns [256 s, 256 s + 128) for S (P aliases the first
// 64) and [256 s + 128, 256 s + 128 + d) for the O accumulator.
//
// Work split: each CTA takes a contiguous range of tiles whose estimated cost
// (longest row of the tile plus one step) sums to 1/grid of the total, so a
// few very long rows (the global rows of the local+global pattern) do not
// leave one SM finishing late; the CTA's two slots take tiles from that range
// in turn through a shared-memory counter.
#pragma once

#include "bsa_common.cuh"

namespace bsa {
namespace rows {

constexpr int kThreads = 384;
constexpr int kSlots = 2;
constexpr int kRegsSoftmax = 216;   // warpgroups 0 and 1
constexpr int kRegsOther = 72;      // warpgroup 2 (producers, MMA issuers)
constexpr int kRegsAtLaunch = 168;  // 65536 / 384 rounded down to a multiple of 8
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kThreads * kRegsAtLaunch,
              "register split exceeds the registers the CTA is launched with");

template <int BS, int D>
struct Cfg {
  static constexpr int TM = 128;                 // query rows per tile
  static constexpr int R = TM / BS;              // block rows per tile
  static constexpr int NK = 128;                 // keys per step
  static constexpr int BPS = NK / BS;            // blocks per step
  static constexpr int KATOMS = D / 64;          // 128-byte column atoms of a D-wide row
  static constexpr int Q_BYTES = TM * D * 2;
  static constexpr int CH_BYTES = NK * D * 2;    // one K or V stage
  static constexpr int NKS = D == 64 ? 2 : 1;    // K stages per slot
  static constexpr int NVS = D == 64 ? 2 : 1;    // V stages per slot
  static constexpr int SLOT_KV = (NKS + NVS) * CH_BYTES;
  static constexpr int OFF_Q = 0;                // + slot * Q_BYTES
  static constexpr int OFF_KV = kSlots * Q_BYTES;  // + slot * SLOT_KV: K stages, then V stages
  static constexpr int OFF_CTRL = OFF_KV + kSlots * SLOT_KV;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TMEM_SLOT = 256;
  static constexpr uint32_t TMEM_O = 128;
  static_assert((Q_BYTES % 1024) == 0 && (CH_BYTES % 1024) == 0, "1024-byte aligned stages");
};

struct SlotCtrl {
  uint64_t bm_full[2], bm_empty[2];
  uint64_t q_full, q_empty;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full, p_full, o_full, o_empty;
  uint64_t final_bar;
  long long tile[2];  // tile index of each bitmap buffer, -1 = no more work
  int n[2];           // union size (blocks) of each bitmap buffer
};

struct Ctrl {
  SlotCtrl slot[kSlots];
  long long range_begin, range_end;
  long long scan[kThreads / 32];
  int next_tile;
  uint32_t tmem_base;
  AbortFlag abort;
  uint32_t bitmap[kSlots][2][5 * kMaxBitmapWords];  // R block-row maps, then their union
};

// Estimated cost of tile group (h, g) in blocks: the longest of its rows, plus
// one step for the per-tile overhead.
template <int BS>
__device__ __forceinline__ long long group_cost(const FwdArgs& a, long long hg) {
  constexpr int R = 128 / BS;
  const long long h = hg / a.G;
  const int g = static_cast<int>(hg - h * a.G);
  const int32_t* rp = a.row_ptr + h * a.M;
  int mx = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int r = g * R + i;
    if (r < a.M) mx = max(mx, __ldg(rp + r + 1) - __ldg(rp + r));
  }
  return mx + R;
}

// All threads: the contiguous tile range [range_begin, range_end) of this CTA.
// Tile T = (b*H + h)*G + g has prefix cost b*P + p(h*G + g), p the exclusive
// prefix of group_cost over the H*G groups of one batch element and P their
// sum; CTA c owns the tiles whose prefix lies in [c*total/grid, (c+1)*total/grid).
template <int BS>
__device__ void compute_range(const FwdArgs& a, Ctrl* ctl) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long HG = static_cast<long long>(a.H) * a.G;
  const long long seg = (HG + kThreads - 1) / kThreads;
  const long long lo = min(HG, tid * seg), hi = min(HG, lo + seg);
  long long sum = 0;
  for (long long hg = lo; hg < hi; ++hg) sum += group_cost<BS>(a, hg);
  long long incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) ctl->scan[warp] = incl;
  __syncthreads();
  long long base = 0, per_b = 0;
  for (int w = 0; w < kThreads / 32; ++w) {
    if (w < warp) base += ctl->scan[w];
    per_b += ctl->scan[w];
  }
  const long long excl = base + incl - sum;
  const long long nb = a.num_tiles / HG;
  const long long total = per_b * nb;
  const long long grid = gridDim.x;
  for (int e = 0; e < 2; ++e) {
    const long long c = static_cast<long long>(blockIdx.x) + e;
    const long long x = (total / grid) * c + ((total % grid) * c) / grid;
    long long* out = e == 0 ? &ctl->range_begin : &ctl->range_end;
    if (x >= total) {
      if (tid == 0) *out = a.num_tiles;
      continue;
    }
    const long long b = x / per_b, rem = x - b * per_b;
    if (rem == 0) {
      if (tid == 0) *out = b * HG;
      continue;
    }
    if (excl < rem && rem <= excl + sum) {
      long long run = excl, hg = lo;
      while (run < rem) run += group_cost<BS>(a, hg++);
      *out = b * HG + hg;
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------ producer warp
template <int BS, int D>
__device__ void load_role(int s, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                          const CUtensorMap* tmV, const FwdArgs& a, uint8_t* smem, Ctrl* ctl) {
  using C = Cfg<BS, D>;
  SlotCtrl& sc = ctl->slot[s];
  const int lane = threadIdx.x & 31;
  uint8_t* q_s = smem + C::OFF_Q + s * C::Q_BYTES;
  uint8_t* k_s = smem + C::OFF_KV + s * C::SLOT_KV;
  uint8_t* v_s = k_s + C::NKS * C::CH_BYTES;
  uint32_t q_loads = 0, k_loads = 0, v_loads = 0;
  bool ok = true;
  if (lane == 0) {
    prefetch_tensormap(tmQ);
    prefetch_tensormap(tmK);
    prefetch_tensormap(tmV);
  }
  for (int t = 0;; ++t) {
    const int buf = t & 1;
    int w_ok = 1;
    long long tile = -1;
    if (lane == 0) {
      w_ok = wait_bounded(&sc.bm_empty[buf], ((t >> 1) & 1) ^ 1, &ctl->abort);
      if (w_ok) {
        tile = ctl->range_begin + atomicAdd(&ctl->next_tile, 1);
        if (tile >= ctl->range_end) tile = -1;
      }
    }
    if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
    tile = __shfl_sync(0xffffffffu, tile, 0);

    uint32_t* bm = ctl->bitmap[s][buf];
    const int W = a.W;
    long long bh = 0;
    int n = 0;
    if (tile >= 0) {
      for (int w = lane; w < (C::R + 1) * W; w += 32) bm[w] = 0u;
      __syncwarp();
      bh = tile / a.G;
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
          if (a.causal && j > r) continue;  // every key of the block is after every query
          atomicOr(&bm[i * W + (j >> 5)], 1u << (j & 31));
          atomicOr(&bm[C::R * W + (j >> 5)], 1u << (j & 31));
        }
      }
      __threadfence_block();
      __syncwarp();
      n = union_count(bm + C::R * W, W);
    }
    if (lane == 0) {
      sc.tile[buf] = tile;
      sc.n[buf] = n;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sc.bm_full[buf]);
    if (tile < 0) break;
    if (n == 0) continue;

    if (lane == 0) {
      const int g = static_cast<int>(tile - bh * a.G);
      ok = wait_bounded(&sc.q_empty, (q_loads & 1) ^ 1, &ctl->abort);
      if (ok) {
        mbar_arrive_expect_tx(&sc.q_full, C::Q_BYTES);
#pragma unroll
        for (int ka = 0; ka < C::KATOMS; ++ka)
          tma_load_3d(q_s + ka * (C::TM * 128), tmQ, &sc.q_full, ka * 64, g * C::TM,
                      static_cast<int>(bh));
        ++q_loads;
      }
      BitIter it(bm + C::R * W, W);
      const int steps = (n + C::BPS - 1) / C::BPS;
      for (int j = 0; ok && j < steps; ++j) {
        int row0[C::BPS];  // first token of each block of the step; N (all out of range) pads
#pragma unroll
        for (int b = 0; b < C::BPS; ++b) {
          const int jb = it.next();
          row0[b] = jb >= 0 ? jb * BS : a.N;
        }
        const uint32_t ks = k_loads % C::NKS;
        ok = wait_bounded(&sc.k_empty[ks], ((k_loads / C::NKS) & 1) ^ 1, &ctl->abort);
        if (!ok) break;
        mbar_arrive_expect_tx(&sc.k_full[ks], C::CH_BYTES);
#pragma unroll
        for (int b = 0; b < C::BPS; ++b)
#pragma unroll
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_load_3d(k_s + ks * C::CH_BYTES + ka * (C::NK * 128) + b * (BS * 128), tmK,
                        &sc.k_full[ks], ka * 64, row0[b], static_cast<int>(bh));
        ++k_loads;
        const uint32_t vs = v_loads % C::NVS;
        ok = wait_bounded(&sc.v_empty[vs], ((v_loads / C::NVS) & 1) ^ 1, &ctl->abort);
        if (!ok) break;
        mbar_arrive_expect_tx(&sc.v_full[vs], C::CH_BYTES);
#pragma unroll
        for (int b = 0; b < C::BPS; ++b)
#pragma unroll
          for (int ka = 0; ka < C::KATOMS; ++ka)
            tma_load_3d(v_s + vs * C::CH_BYTES + ka * (C::NK * 128) + b * (BS * 128), tmV,
                        &sc.v_full[vs], ka * 64, row0[b], static_cast<int>(bh));
        ++v_loads;
      }
    }
    if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { ok = false; break; }
  }
  // On an early exit, let every copy already issued land before the CTA ends.
  if (!ok && lane == 0) {
    if (q_loads > 0) wait_drain(&sc.q_full, (q_loads - 1) & 1);
    for (uint32_t st = 0; st < C::NKS; ++st)
      if (k_loads > st) {
        const uint32_t last = st + C::NKS * ((k_loads - 1 - st) / C::NKS);
        wait_drain(&sc.k_full[st], (last / C::NKS) & 1);
      }
    for (uint32_t st = 0; st < C::NVS; ++st)
      if (v_loads > st) {
        const uint32_t last = st + C::NVS * ((v_loads - 1 - st) / C::NVS);
        wait_drain(&sc.v_full[st], (last / C::NVS) & 1);
      }
  }
  __syncwarp();
}

// ---------------------------------------------------------------- MMA issuer
// Per step: S = Q K^T, then (once the softmax has written P) O += P V.  The
// QK of the next step is issued right after the PV of this one: MMAs of one
// thread run in issue order, so it overwrites S/P only after the PV read P,
// and the commit that reports it also reports that PV.
template <int BS, int D>
__device__ void mma_role(int s, const FwdArgs& a, uint8_t* smem, Ctrl* ctl, uint32_t tmem) {
  using C = Cfg<BS, D>;
  SlotCtrl& sc = ctl->slot[s];
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, C::NK, false, false);  // Q, K K-major
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);       // V MN-major
  const uint32_t q_base = smem_u32(smem + C::OFF_Q + s * C::Q_BYTES);
  const uint32_t k_base = smem_u32(smem + C::OFF_KV + s * C::SLOT_KV);
  const uint32_t v_base = k_base + C::NKS * C::CH_BYTES;
  const uint32_t t_s = tmem + s * C::TMEM_SLOT;
  const uint32_t t_o = t_s + C::TMEM_O;
  uint32_t k_cons = 0, v_cons = 0, q_uses = 0, p_seen = 0, o_tiles = 0;
  bool ok = true;
  for (int t = 0; ok; ++t) {
    const int buf = t & 1;
    if (!wait_bounded(&sc.bm_full[buf], (t >> 1) & 1, &ctl->abort)) break;
    const long long tile = sc.tile[buf];
    const int n = sc.n[buf];
    mbar_arrive(&sc.bm_empty[buf]);
    if (tile < 0) break;
    if (n == 0) continue;
    const int steps = (n + C::BPS - 1) / C::BPS;
    if (!wait_bounded(&sc.q_full, q_uses & 1, &ctl->abort)) break;
    ++q_uses;
    for (int j = 0; j < steps; ++j) {
      const uint32_t ks = k_cons % C::NKS;
      if (!wait_bounded(&sc.k_full[ks], (k_cons / C::NKS) & 1, &ctl->abort)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t ad = sdesc_sw128(q_base + (kk >> 2) * (C::TM * 128) + (kk & 3) * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(
            k_base + ks * C::CH_BYTES + (kk >> 2) * (C::NK * 128) + (kk & 3) * 32, 16, 1024);
        umma_bf16_ss(t_s, ad, bd, kIdescQK, kk > 0 ? 1u : 0u);
      }
      umma_commit(&sc.k_empty[ks]);
      umma_commit(&sc.s_full);
      if (j == steps - 1) umma_commit(&sc.q_empty);
      ++k_cons;

      if (!wait_bounded(&sc.p_full, p_seen & 1, &ctl->abort)) { ok = false; break; }
      ++p_seen;
      const uint32_t vs = v_cons % C::NVS;
      if (!wait_bounded(&sc.v_full[vs], (v_cons / C::NVS) & 1, &ctl->abort)) { ok = false; break; }
      if (j == 0 && o_tiles > 0 &&
          !wait_bounded(&sc.o_empty, (o_tiles - 1) & 1, &ctl->abort)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < C::NK / 16; ++kk) {
        const uint64_t bd =
            sdesc_sw128(v_base + vs * C::CH_BYTES + kk * (16 * 128), C::NK * 128, 1024);
        umma_bf16_ts(t_o, t_s + kk * 8, bd, kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&sc.v_empty[vs]);
      ++v_cons;
      if (j == steps - 1) umma_commit(&sc.o_full);
    }
    ++o_tiles;
  }
  // Every MMA issued must complete before the TMEM is released.
  umma_commit(&sc.final_bar);
  wait_drain(&sc.final_bar, 0);
}

// ------------------------------------------------------------ softmax warps
template <int BS, int D>
__device__ void softmax_role(int s, const FwdArgs& a, Ctrl* ctl, uint32_t tmem) {
  using C = Cfg<BS, D>;
  SlotCtrl& sc = ctl->slot[s];
  const int row = threadIdx.x - s * 128;  // query row of the tile
  const int warp = row >> 5;
  const int lane = row & 31;
  const int sub = row / BS;               // block row of the tile this thread belongs to
  const int qq = row % BS;                // position inside that block row
  const uint32_t t_s = tmem + s * C::TMEM_SLOT + (static_cast<uint32_t>(warp * 32) << 16);
  const uint32_t t_o = t_s + C::TMEM_O;
  const float sl2 = a.scale_log2;
  constexpr float kNegInf = -INFINITY;
  uint32_t s_seen = 0, o_seen = 0;

  for (int t = 0;; ++t) {
    const int buf = t & 1;
    if (!warp_wait(&sc.bm_full[buf], (t >> 1) & 1, &ctl->abort)) return;
    const long long tile = sc.tile[buf];
    const int n = sc.n[buf];
    if (tile < 0) return;
    const uint32_t* bm = ctl->bitmap[s][buf];
    const uint32_t* mine = bm + sub * a.W;
    const long long bh = tile / a.G;
    const int g = static_cast<int>(tile - bh * a.G);
    const int r_sub = g * C::R + sub;
    const bool row_ok = r_sub < a.M;
    const int steps = (n + C::BPS - 1) / C::BPS;

    float m_used = kNegInf;  // running max, log2 units of the scaled score
    float l = 0.f;           // running sum of 2^(s - m_used)
    BitIter it(bm + C::R * a.W, a.W);
    for (int j = 0; j < steps; ++j) {
      int jb[C::BPS];
      bool val[C::BPS];
      bool any = false;
#pragma unroll
      for (int b = 0; b < C::BPS; ++b) {
        jb[b] = it.next();
        val[b] = row_ok && jb[b] >= 0 && ((mine[jb[b] >> 5] >> (jb[b] & 31)) & 1u);
        any = any || val[b];
      }
      if (!warp_wait(&sc.s_full, s_seen & 1, &ctl->abort)) return;
      ++s_seen;
      tc_fence_after();
      uint32_t x[128];
      if (any) {
        // All four column groups are loaded even when some blocks are masked:
        // a conditional tcgen05.ld leaves its registers undefined on one path,
        // which makes the compiler spill the whole score row.
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(t_s + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&x[c * 32]));
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&x[c * 32]));

        float mx = kNegInf;
#pragma unroll
        for (int b = 0; b < C::BPS; ++b) {
          if (!val[b]) continue;
          const bool diag = a.causal && jb[b] == r_sub;
#pragma unroll
          for (int c = 0; c < BS; ++c) {
            float v = __uint_as_float(x[b * BS + c]) * sl2;
            if (diag && c > qq) v = kNegInf;  // key after the query (diagonal block only)
            x[b * BS + c] = __float_as_uint(v);
            mx = fmaxf(mx, v);
          }
        }
        float factor = 1.f;
        bool need_rescale = false;
        const float m_new = fmaxf(m_used, mx);
        if (m_new > m_used + kRescaleThreshold) {
          if (l > 0.f) {
            need_rescale = true;
            factor = ex2_approx(m_used - m_new);
          }
          m_used = m_new;
        }
        // The commit behind s_full also covers the previous PV: O is final here.
        if (__any_sync(0xffffffffu, need_rescale)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t u[32];
            tmem_ld32(t_o + c * 32, u);
            tmem_wait_ld();
            reg_fence32(u);
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * factor);
            tmem_st32(t_o + c * 32, u);
          }
        }
        const float mu = m_used == kNegInf ? 0.f : m_used;
        float rs = 0.f;
#pragma unroll
        for (int b = 0; b < C::BPS; ++b) {
#pragma unroll
          for (int c = 0; c < BS; ++c) {
            float p = 0.f;
            if (val[b]) {
              p = ex2_approx(__uint_as_float(x[b * BS + c]) - mu);
              rs += p;
            }
            x[b * BS + c] = __float_as_uint(p);
          }
        }
        l = l * factor + rs;
#pragma unroll
        for (int i = 0; i < 64; ++i)
          x[i] = pack_bf16x2(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) x[i] = 0u;
      }
      tmem_st32(t_s, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
      tmem_st32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sc.p_full);
    }

    // Epilogue: O / l in bf16 and LSE = (m + log2 l) ln 2.
    const long long qtok = static_cast<long long>(g) * C::TM + row;
    __nv_bfloat16* orow = a.O + (bh * a.N + qtok) * D;
    if (n > 0) {
      if (!warp_wait(&sc.o_full, o_seen & 1, &ctl->abort)) return;
      ++o_seen;
      tc_fence_after();
      uint32_t o[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(t_o + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&o[c * 32]));
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&o[c * 32]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sc.o_empty);
      if (row_ok) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[c * 8 + 0]) * inv, __uint_as_float(o[c * 8 + 1]) * inv);
          v.y = pack_bf16x2(__uint_as_float(o[c * 8 + 2]) * inv, __uint_as_float(o[c * 8 + 3]) * inv);
          v.z = pack_bf16x2(__uint_as_float(o[c * 8 + 4]) * inv, __uint_as_float(o[c * 8 + 5]) * inv);
          v.w = pack_bf16x2(__uint_as_float(o[c * 8 + 6]) * inv, __uint_as_float(o[c * 8 + 7]) * inv);
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
    if (lane == 0) mbar_arrive(&sc.bm_empty[buf]);
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
    for (int s = 0; s < kSlots; ++s) {
      SlotCtrl& sc = ctl->slot[s];
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sc.bm_full[b], 1);
        mbar_init(&sc.bm_empty[b], 5);  // four softmax warps + the MMA issuer
        mbar_init(&sc.k_full[b], 1);
        mbar_init(&sc.k_empty[b], 1);
        mbar_init(&sc.v_full[b], 1);
        mbar_init(&sc.v_empty[b], 1);
      }
      mbar_init(&sc.q_full, 1);
      mbar_init(&sc.q_empty, 1);
      mbar_init(&sc.s_full, 1);
      mbar_init(&sc.p_full, 4);
      mbar_init(&sc.o_full, 1);
      mbar_init(&sc.o_empty, 4);
      mbar_init(&sc.final_bar, 1);
    }
    ctl->next_tile = 0;
    ctl->abort.v = 0;
    fence_mbar_init();
  }
  if (warp == 10) {
    tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  compute_range<BS>(args, ctl);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp < 8) {
    setmaxnreg_inc<kRegsSoftmax>();
    softmax_role<BS, D>(warp >> 2, args, ctl, tmem);
    __syncwarp();
  } else {
    setmaxnreg_dec<kRegsOther>();
    if (warp < 10) {
      load_role<BS, D>(warp - 8, &tmQ, &tmK, &tmV, args, smem, ctl);
    } else {
      if ((threadIdx.x & 31) == 0) mma_role<BS, D>(warp - 10, args, smem, ctl, tmem);
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 10) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace rows
}  // namespace bsa
