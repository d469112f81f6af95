// ep_plan.h -- where the routed rows of an expert-parallel layer go.
//
// Expert parallelism (DeepSeek-V3 technical report summary, section 3.1 "Compute
// Clusters" and section 3.2.1, the all-to-all dispatch and combine): the mN routed
// experts are split over G ranks in equal contiguous ranges (expert e lives on rank
// e / (mN / G)); every rank routes its own tokens, sends each (token, slot) row to the
// rank that holds the slot's expert, and sums the rows that come back.
//
// The receiving rank's row buffer has the single-GPU layout of its own experts: the
// rows of local expert l are contiguous, start at row_start[l], and each expert's
// segment is padded to a multiple of kEpRowAlign rows (the grouped GEMMs' 256-row
// pair tiles).  Within an expert the rows come in ascending sending rank, and within
// one sender in that sender's own order (ascending token id), so the owner's rows of
// expert e are those of a stable counting sort of the concatenated batch
// [rank 0's tokens, rank 1's tokens, ...] restricted to e.
//
// Every function reads the per-rank counts through cnt[r][e] (expert e's rows on
// rank r, e a global expert id) and is plain arithmetic; the device kernel and the
// host entry point moe_ep_plan both call them.
#pragma once

#include <cstdint>

#ifdef __CUDACC__
#define FGS_HD __host__ __device__
#else
#define FGS_HD
#endif

namespace fgs {

constexpr int kEpMaxRanks = 32;
constexpr int kEpRowAlign = 256;

FGS_HD inline int32_t ep_pad(int32_t rows) { return (rows + kEpRowAlign - 1) / kEpRowAlign * kEpRowAlign; }

// rows of global expert e over all ranks
FGS_HD inline int32_t ep_total(const int32_t* const* cnt, int G, int e) {
  int32_t n = 0;
  for (int r = 0; r < G; ++r) n += cnt[r][e];
  return n;
}

// The first row, in the buffer of the rank that holds global expert e, of the rows that
// rank `sender` sends to e.
FGS_HD inline int32_t ep_dest_base(const int32_t* const* cnt, int G, int N, int sender, int e) {
  const int per = N / G;
  const int first = e / per * per;
  int32_t row = 0;
  for (int f = first; f < e; ++f) row += ep_pad(ep_total(cnt, G, f));
  for (int r = 0; r < sender; ++r) row += cnt[r][e];
  return row;
}

// Rank `owner`'s tables for its local expert l, 0 <= l <= N / G (l = N / G: the totals):
// rows received, first row (padded prefix), prefix of ceil(rows / 256) and of ceil(rows / 128).
FGS_HD inline void ep_owner_entry(const int32_t* const* cnt, int G, int N, int owner, int l, int32_t* count,
                                  int32_t* row_start, int32_t* mtile_start, int32_t* mtile128_start) {
  const int per = N / G;
  const int first = owner * per;
  int32_t rs = 0, mt = 0, m128 = 0;
  for (int f = first; f < first + l; ++f) {
    const int32_t n = ep_total(cnt, G, f);
    rs += ep_pad(n);
    mt += (n + kEpRowAlign - 1) / kEpRowAlign;
    m128 += (n + 127) / 128;
  }
  *count = l < per ? ep_total(cnt, G, first + l) : 0;
  *row_start = rs;
  *mtile_start = mt;
  *mtile128_start = m128;
}

}  // namespace fgs
