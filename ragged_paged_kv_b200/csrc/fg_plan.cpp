#include "fg_plan.h"

#include <algorithm>
#include <cstring>

namespace fg {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

void Plan::pack(void* dst) const {
  char* p = static_cast<char*>(dst);
  if (n_general) std::memcpy(p + off_general, general.data(), general.size() * sizeof(WorkItem));
  if (n_decode) std::memcpy(p + off_decode, decode.data(), decode.size() * sizeof(WorkItem));
  if (n_tc) std::memcpy(p + off_tc, tc.data(), tc.size() * sizeof(WorkItem));
  if (n_dtc) std::memcpy(p + off_dtc, dtc.data(), dtc.size() * sizeof(WorkItem));
  if (n_combine) std::memcpy(p + off_combine, combine.data(), combine.size() * sizeof(CombineItem));
}

void build_plan(const std::vector<int32_t>& q_lens, const std::vector<int32_t>& ctx_lens,
                int n_kv_heads, int g, int head_dim, int window, bool use_tc, Plan* out) {
  (void)head_dim;
  Plan& P = *out;
  P.general.clear();
  P.decode.clear();
  P.tc.clear();
  P.dtc.clear();
  P.combine.clear();
  P.part_rows = 0;
  P.max_combine_rows = 0;
  const int tok_per_tile = std::max(1, kGeneralRows / g);
  const int S = (int)q_lens.size();
  // Append units for one (seq, kv head, token tile) over keys [kb, ke) to
  // `list`, split on `split`-key boundaries of absolute position.
  auto emit = [&](std::vector<WorkItem>& list, int s, int h, int t0, int nt, int kb, int ke,
                  int split) {
    const int R = nt * g;
    const int kb_al = kb - (kb % 64);
    const int n = (ke - kb_al + split - 1) / split;
    if (n <= 1) {
      list.push_back(WorkItem{s, h, t0, nt, kb, ke, -1, R});
      return;
    }
    const int base = P.part_rows;
    for (int i = 0; i < n; ++i) {
      const int lo = i == 0 ? kb : kb_al + i * split;
      const int hi = std::min(ke, kb_al + (i + 1) * split);
      list.push_back(WorkItem{s, h, t0, nt, lo, hi, base + i * R, R});
    }
    P.part_rows += n * R;
    P.combine.push_back(CombineItem{s, h, t0, nt, base, n, R, 0});
    P.max_combine_rows = std::max(P.max_combine_rows, R);
  };
  for (int s = 0; s < S; ++s) {
    const int q = q_lens[s], c = ctx_lens[s];
    if (use_tc && q == 1 && head_dim == 128 && g <= kDtcMaxGroup) {
      const int kb = window > 0 ? std::max(0, c - window + 1) : 0;
      for (int h = 0; h < n_kv_heads; ++h) emit(P.dtc, s, h, 0, 1, kb, c + 1, kTcDecodeSplitKeys);
      continue;
    }
    if (q == 1 && g == 1) {
      const int kb = window > 0 ? std::max(0, c - window + 1) : 0;
      for (int h = 0; h < n_kv_heads; ++h) emit(P.decode, s, h, 0, 1, kb, c + 1, kDecodeSplitKeys);
      continue;
    }
    if (use_tc) {
      const int tpt = kTcRows / g;
      for (int t0 = 0; t0 < q; t0 += tpt) {
        const int nt = std::min(tpt, q - t0);
        const int p0 = c + t0, p1 = c + t0 + nt - 1;
        const int kb = window > 0 ? std::max(0, p0 - window + 1) : 0;
        const int split = nt * g <= 16 ? kTcDecodeSplitKeys : (1 << 30);
        for (int h = 0; h < n_kv_heads; ++h) emit(P.tc, s, h, t0, nt, kb, p1 + 1, split);
      }
      continue;
    }
    for (int t0 = 0; t0 < q; t0 += tok_per_tile) {
      const int nt = std::min(tok_per_tile, q - t0);
      const int p0 = c + t0, p1 = c + t0 + nt - 1;
      const int kb = window > 0 ? std::max(0, p0 - window + 1) : 0;
      for (int h = 0; h < n_kv_heads; ++h) emit(P.general, s, h, t0, nt, kb, p1 + 1, kSplitKeys);
    }
  }
  // longest units first, so the hardware block scheduler ends the grid evenly
  std::stable_sort(P.decode.begin(), P.decode.end(), [](const WorkItem& a, const WorkItem& b) {
    return a.key_end - a.key_begin > b.key_end - b.key_begin;
  });
  auto longest_first = [](const WorkItem& a, const WorkItem& b) {
    return a.key_end - a.key_begin > b.key_end - b.key_begin;
  };
  std::stable_sort(P.tc.begin(), P.tc.end(), longest_first);
  std::stable_sort(P.dtc.begin(), P.dtc.end(), longest_first);
  P.n_general = (int32_t)P.general.size();
  P.n_decode = (int32_t)P.decode.size();
  P.n_tc = (int32_t)P.tc.size();
  P.n_dtc = (int32_t)P.dtc.size();
  P.n_combine = (int32_t)P.combine.size();
  P.off_general = 0;
  P.off_decode = align_up(P.general.size() * sizeof(WorkItem), 256);
  P.off_tc = align_up(P.off_decode + P.decode.size() * sizeof(WorkItem), 256);
  P.off_dtc = align_up(P.off_tc + P.tc.size() * sizeof(WorkItem), 256);
  P.off_combine = align_up(P.off_dtc + P.dtc.size() * sizeof(WorkItem), 256);
  P.total = align_up(P.off_combine + P.combine.size() * sizeof(CombineItem), 256);
}

}  // namespace fg
