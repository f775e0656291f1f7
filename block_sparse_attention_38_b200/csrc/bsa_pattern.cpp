// bsa_pattern.cpp -- host-side block-pattern builder and CSR validator.
//
// Integer work only.  Produces the per-block-row column lists that the
// forward kernel walks ("Block Sparse Attention with Log-Linear Complexity",
// section 3.2: the index table is generated on the CPU before the launch, so
// the kernel never evaluates the pattern rules with per-element branches).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <vector>

#include "bsa.h"

namespace {

// SplitMix64 (Steele, Lea, Flood, OOPSLA 2014) evaluated at an arbitrary
// position of the stream: state after n increments is seed + n * gamma, and
// the output is that state through the variant-13 finaliser.
inline uint64_t splitmix64_at(uint64_t seed, uint64_t n) {
  uint64_t z = seed + n * 0x9E3779B97F4A7C15ull;
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}

inline bool bernoulli_keep(const bsa_pattern_desc& d, int64_t h, int64_t i, int64_t j) {
  if (i == j) return true;  // diagonal forced on: no empty row
  const uint64_t key = static_cast<uint64_t>((h * d.M + i) * d.M + j);
  const uint64_t top53 = splitmix64_at(d.seed, key + 1) >> 11;
  const double u = static_cast<double>(top53) * (1.0 / 9007199254740992.0);  // 2^-53
  return u < d.p;
}

// BigBird random column r of block row i, head h (draws with replacement).
inline int32_t bigbird_column(const bsa_pattern_desc& d, int64_t h, int64_t i, int64_t r) {
  const uint64_t key = static_cast<uint64_t>((h * d.M + i) * d.num_random + r);
  const uint64_t top53 = splitmix64_at(d.seed, key + 1) >> 11;
  const double u = static_cast<double>(top53) * (1.0 / 9007199254740992.0);  // 2^-53
  const int64_t j = static_cast<int64_t>(u * d.M);
  return static_cast<int32_t>(j < d.M ? j : d.M - 1);
}

// Appends the columns of block row i (head h) to out, ascending and distinct.
void row_columns(const bsa_pattern_desc& d, int32_t h, int32_t i, std::vector<int32_t>& out,
                 std::vector<int32_t>& tmp) {
  const int32_t M = d.M;
  tmp.clear();
  switch (d.kind) {
    case BSA_LOGLINEAR: {
      const int64_t lo = std::max<int64_t>(0, int64_t(i) - d.local_radius);
      const int64_t hi = std::min<int64_t>(M - 1, int64_t(i) + d.local_radius);
      for (int64_t j = lo; j <= hi; ++j) tmp.push_back(static_cast<int32_t>(j));
      for (int32_t k = 0; k <= d.log_kmax; ++k) {
        const int64_t s = int64_t(1) << k;
        if (i - s >= 0) tmp.push_back(static_cast<int32_t>(i - s));
        if (i + s < M) tmp.push_back(static_cast<int32_t>(i + s));
      }
      for (int32_t a = 0; a < d.n_anchors; ++a) tmp.push_back(d.anchors[a]);
      break;
    }
    case BSA_LOCAL_GLOBAL: {
      bool global_row = false;
      for (int32_t a = 0; a < d.n_anchors; ++a) global_row |= (d.anchors[a] == i);
      if (global_row) {
        for (int32_t j = 0; j < M; ++j) tmp.push_back(j);
      } else {
        const int64_t lo = std::max<int64_t>(0, int64_t(i) - d.local_radius);
        const int64_t hi = std::min<int64_t>(M - 1, int64_t(i) + d.local_radius);
        for (int64_t j = lo; j <= hi; ++j) tmp.push_back(static_cast<int32_t>(j));
        for (int32_t a = 0; a < d.n_anchors; ++a) tmp.push_back(d.anchors[a]);
      }
      break;
    }
    case BSA_BERNOULLI: {
      for (int32_t j = 0; j < M; ++j)
        if (bernoulli_keep(d, h, i, j)) tmp.push_back(j);
      break;
    }
    case BSA_SLIDING_WINDOW: {
      const int64_t lo = std::max<int64_t>(0, int64_t(i) - d.local_radius);
      const int64_t hi = std::min<int64_t>(M - 1, int64_t(i) + d.local_radius);
      for (int64_t j = lo; j <= hi; ++j)
        if ((int64_t(i) - j) % d.dilation == 0) tmp.push_back(static_cast<int32_t>(j));
      break;
    }
    case BSA_BIGBIRD: {
      bool global_row = false;
      for (int32_t a = 0; a < d.n_anchors; ++a) global_row |= (d.anchors[a] == i);
      if (global_row) {
        for (int32_t j = 0; j < M; ++j) tmp.push_back(j);
      } else {
        const int64_t lo = std::max<int64_t>(0, int64_t(i) - d.local_radius);
        const int64_t hi = std::min<int64_t>(M - 1, int64_t(i) + d.local_radius);
        for (int64_t j = lo; j <= hi; ++j) tmp.push_back(static_cast<int32_t>(j));
        for (int32_t a = 0; a < d.n_anchors; ++a) tmp.push_back(d.anchors[a]);
        for (int32_t r = 0; r < d.num_random; ++r) tmp.push_back(bigbird_column(d, h, i, r));
      }
      break;
    }
    default:
      break;
  }
  std::sort(tmp.begin(), tmp.end());
  tmp.erase(std::unique(tmp.begin(), tmp.end()), tmp.end());
  for (int32_t j : tmp) {
    if (j < 0 || j >= M) continue;
    if (d.causal && j > i) continue;
    out.push_back(j);
  }
}

bool desc_ok(const bsa_pattern_desc* d) {
  if (!d) return false;
  if (d->M < 1 || d->H < 1) return false;
  if (d->kind < BSA_LOGLINEAR || d->kind > BSA_BIGBIRD) return false;
  if (d->local_radius < 0) return false;
  if (d->kind == BSA_LOGLINEAR && (d->log_kmax < 0 || d->log_kmax > 30)) return false;
  if (d->kind == BSA_BERNOULLI && !(d->p >= 0.0 && d->p <= 1.0)) return false;
  if (d->n_anchors < 0 || (d->n_anchors > 0 && d->anchors == nullptr)) return false;
  if (d->causal != 0 && d->causal != 1) return false;
  if (d->kind == BSA_SLIDING_WINDOW && d->dilation < 1) return false;
  if (d->kind == BSA_BIGBIRD && d->num_random < 0) return false;
  return true;
}

}  // namespace

extern "C" int bsa_build_pattern(const bsa_pattern_desc* desc, int32_t* row_ptr,
                                 int32_t* col_idx, int64_t cap, int64_t* nnz_out) {
  if (!desc_ok(desc) || nnz_out == nullptr) return BSA_ERR_INVALID_ARG;
  if ((row_ptr == nullptr) != (col_idx == nullptr)) return BSA_ERR_INVALID_ARG;
  const bsa_pattern_desc& d = *desc;
  const int64_t rows = int64_t(d.H) * d.M;
  if (rows + 1 > INT32_MAX) return BSA_ERR_INVALID_ARG;

  // Heads repeat for the deterministic kinds; Bernoulli and BigBird draw per head.
  const bool per_head = d.kind == BSA_BERNOULLI || (d.kind == BSA_BIGBIRD && d.num_random > 0);
  const int32_t distinct_heads = per_head ? d.H : 1;
  std::vector<int32_t> cols, tmp;
  std::vector<int64_t> head_ptr;  // row offsets inside cols for the distinct heads
  head_ptr.reserve(size_t(distinct_heads) * d.M + 1);
  head_ptr.push_back(0);
  for (int32_t h = 0; h < distinct_heads; ++h)
    for (int32_t i = 0; i < d.M; ++i) {
      row_columns(d, h, i, cols, tmp);
      head_ptr.push_back(static_cast<int64_t>(cols.size()));
    }
  const int64_t per_pass = static_cast<int64_t>(cols.size());
  const int64_t nnz = (distinct_heads == d.H) ? per_pass : per_pass * d.H;
  if (nnz > INT32_MAX) return BSA_ERR_INVALID_ARG;
  *nnz_out = nnz;
  if (row_ptr == nullptr) return BSA_OK;
  if (cap < nnz) return BSA_ERR_BUFFER_TOO_SMALL;

  int64_t out = 0;
  for (int32_t h = 0; h < d.H; ++h) {
    const int32_t src = (distinct_heads == d.H) ? h : 0;
    for (int32_t i = 0; i < d.M; ++i) {
      const int64_t r = int64_t(h) * d.M + i;
      const int64_t s = int64_t(src) * d.M + i;
      row_ptr[r] = static_cast<int32_t>(out);
      for (int64_t p = head_ptr[s]; p < head_ptr[s + 1]; ++p) col_idx[out++] = cols[p];
    }
  }
  row_ptr[rows] = static_cast<int32_t>(out);
  return BSA_OK;
}

extern "C" int bsa_validate_pattern(const int32_t* row_ptr, const int32_t* col_idx,
                                    int64_t col_cap, int32_t H, int32_t M, int32_t causal) {
  if (row_ptr == nullptr || H < 1 || M < 1 || col_cap < 0) return BSA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return BSA_ERR_INVALID_ARG;
  const int64_t rows = int64_t(H) * M;
  if (row_ptr[0] != 0) return BSA_ERR_BAD_PATTERN;
  for (int64_t r = 0; r < rows; ++r)
    if (row_ptr[r + 1] < row_ptr[r]) return BSA_ERR_BAD_PATTERN;
  if (row_ptr[rows] > col_cap) return BSA_ERR_BUFFER_TOO_SMALL;
  if (row_ptr[rows] > 0 && col_idx == nullptr) return BSA_ERR_INVALID_ARG;
  for (int64_t r = 0; r < rows; ++r) {
    const int32_t i = static_cast<int32_t>(r % M);
    int64_t prev = -1;
    for (int32_t p = row_ptr[r]; p < row_ptr[r + 1]; ++p) {
      const int32_t j = col_idx[p];
      if (j < 0 || j >= M || j <= prev) return BSA_ERR_BAD_PATTERN;
      if (causal && j > i) return BSA_ERR_BAD_PATTERN;
      prev = j;
    }
  }
  return BSA_OK;
}

// Column-major copy of a block-CSR (the backward's dK/dV walk): for each
// (h, column j), the block rows i listing j, ascending; a column repeated
// within a row counts once.  Two passes: count, then fill.
extern "C" int bsa_transpose_pattern(const int32_t* row_ptr, const int32_t* col_idx, int32_t H,
                                     int32_t M, int32_t* col_ptr, int32_t* row_idx,
                                     int64_t cap, int64_t* nnz_out) {
  if (row_ptr == nullptr || col_ptr == nullptr || nnz_out == nullptr || H < 1 || M < 1 ||
      cap < 0)
    return BSA_ERR_INVALID_ARG;
  const int64_t rows = int64_t(H) * M;
  if (row_ptr[0] != 0) return BSA_ERR_BAD_PATTERN;
  for (int64_t r = 0; r < rows; ++r)
    if (row_ptr[r + 1] < row_ptr[r]) return BSA_ERR_BAD_PATTERN;
  if (row_ptr[rows] > 0 && col_idx == nullptr) return BSA_ERR_INVALID_ARG;
  std::vector<int64_t> count(static_cast<size_t>(rows) + 1, 0);
  for (int64_t e = 0; e < row_ptr[rows]; ++e)
    if (col_idx[e] < 0 || col_idx[e] >= M) return BSA_ERR_BAD_PATTERN;
  // count, with a per-row stamp so that repeats within a row count once
  std::vector<int32_t> stamp(static_cast<size_t>(M), -1);  // last row that listed column j
  for (int64_t r = 0; r < rows; ++r) {
    const int64_t h = r / M;
    for (int32_t p = row_ptr[r]; p < row_ptr[r + 1]; ++p) {
      const int32_t j = col_idx[p];
      if (stamp[j] == static_cast<int32_t>(r)) continue;
      stamp[j] = static_cast<int32_t>(r);
      ++count[static_cast<size_t>(h * M + j) + 1];
    }
  }
  for (int64_t c = 0; c < rows; ++c) count[c + 1] += count[c];
  *nnz_out = count[static_cast<size_t>(rows)];
  if (count[static_cast<size_t>(rows)] > cap) return BSA_ERR_BUFFER_TOO_SMALL;
  if (count[static_cast<size_t>(rows)] > INT32_MAX) return BSA_ERR_UNSUPPORTED;
  if (count[static_cast<size_t>(rows)] > 0 && row_idx == nullptr) return BSA_ERR_INVALID_ARG;
  std::vector<int64_t> fill(count.begin(), count.end() - 1);
  std::fill(stamp.begin(), stamp.end(), -1);
  for (int64_t r = 0; r < rows; ++r) {  // rows in ascending order: each column list ascends
    const int64_t h = r / M;
    for (int32_t p = row_ptr[r]; p < row_ptr[r + 1]; ++p) {
      const int32_t j = col_idx[p];
      if (stamp[j] == static_cast<int32_t>(r)) continue;
      stamp[j] = static_cast<int32_t>(r);
      row_idx[fill[static_cast<size_t>(h * M + j)]++] = static_cast<int32_t>(r - h * M);
    }
  }
  for (int64_t c = 0; c <= rows; ++c) col_ptr[c] = static_cast<int32_t>(count[static_cast<size_t>(c)]);
  return BSA_OK;
}

extern "C" int bsa_version(void) { return 200; }  // 0.2.0: top-k, decode, backward
