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
                int n_kv_heads, int g, int head_dim, int window, bool use_tc, int slots, Plan* out) {
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
  // Pieces per dense query tile (the same for all kv heads of a token tile),
  // in emit order; decided before emitting (see below).
  std::vector<int32_t>& dense_pieces = P.sort_tmp_pieces;
  dense_pieces.clear();
  // Append the units of one (seq, token tile) over keys [kb, ke) for every kv
  // head to `list`, split on `split`-key boundaries of absolute position.
  // The split ranges are computed once and repeated per head.
  int32_t rng[2 * 64];
  auto emit = [&](std::vector<WorkItem>& list, int s, int t0, int nt, int kb, int ke, int split) {
    const int R = nt * g;
    const int kb_al = kb - (kb % 64);
    const int n = std::min(64, (ke - kb_al + split - 1) / split);
    if (n <= 1) {
      for (int h = 0; h < n_kv_heads; ++h) list.push_back(WorkItem{s, h, t0, nt, kb, ke, -1, R});
      return;
    }
    const int sp = (ke - kb_al + n - 1) / n;  // never more than 64 pieces
    const int step = std::max(split, (sp + 63) & ~63);
    int m = 0;
    for (int lo = kb; lo < ke; ++m) {
      const int hi = std::min(ke, kb_al + (m + 1) * step);
      rng[2 * m] = lo;
      rng[2 * m + 1] = hi;
      lo = hi;
    }
    for (int h = 0; h < n_kv_heads; ++h) {
      const int base = P.part_rows;
      for (int i = 0; i < m; ++i) list.push_back(WorkItem{s, h, t0, nt, rng[2 * i], rng[2 * i + 1], base + i * R, R});
      P.part_rows += m * R;
      P.combine.push_back(CombineItem{s, h, t0, nt, base, m, R, 0});
    }
    P.max_combine_rows = std::max(P.max_combine_rows, R);
  };
  // Few long query tiles leave persistent CTAs idle at the end. The target
  // is about 4 units per CTA slot: when the dense tiles (x kv heads) are
  // fewer, the longest tiles of at least 2 * kTcMinSplitKeys keys are cut
  // into pieces of at least kTcMinSplitKeys keys, merged by the combine
  // kernel, and only as many as the target needs: P pieces per kv head are
  // spread over the n cut-able tiles as floor(P / n) each, one more for the
  // P % n longest (at most 8 per tile). Splitting only what the balance
  // needs keeps the split partials, which are written in fp32 and merged
  // again, few.
  size_t dense_next = 0;
  if (use_tc) {
    const int tpt = kTcUnitRows / g;
    std::vector<std::pair<int32_t, int32_t>> elig;  // (keys, index in emit order)
    int32_t n_tiles = 0, n_inelig = 0;
    for (int s = 0; s < S; ++s) {
      const int q = q_lens[s], c = ctx_lens[s];
      // the sequences the loop below sends to the decode kernels
      if (q == 1 && ((head_dim == 128 && g <= kDtcMaxGroup) || g == 1)) continue;
      for (int t0 = 0; t0 < q; t0 += tpt, ++n_tiles) {
        const int nt = std::min(tpt, q - t0);
        const int p0 = c + t0, p1 = c + t0 + nt - 1;
        const int kb = window > 0 ? std::max(0, p0 - window + 1) : 0;
        const int nk = p1 + 1 - kb;
        if (nt * g > 16 && nk >= 2 * kTcMinSplitKeys)
          elig.push_back({nk, n_tiles});
        else
          ++n_inelig;
      }
    }
    const long long target = 4LL * slots;
    if (!elig.empty() && (long long)n_tiles * n_kv_heads < target) {
      const long long per_head = (target + n_kv_heads - 1) / n_kv_heads;  // pieces per kv head
      const long long pe = per_head - n_inelig;                            // for the cut-able tiles
      const long long n = (long long)elig.size();
      const long long base = pe / n, rem = pe % n;
      if (base >= 1) {
        std::stable_sort(elig.begin(), elig.end(),
                         [](const std::pair<int32_t, int32_t>& x, const std::pair<int32_t, int32_t>& y) {
                           return x.first > y.first;
                         });
        dense_pieces.assign(n_tiles, 1);
        for (long long i = 0; i < n; ++i)
          dense_pieces[elig[i].second] = (int32_t)std::min<long long>(8, base + (i < rem ? 1 : 0));
      }
    }
  }
  for (int s = 0; s < S; ++s) {
    const int q = q_lens[s], c = ctx_lens[s];
    if (use_tc && q == 1 && head_dim == 128 && g <= kDtcMaxGroup) {
      const int kb = window > 0 ? std::max(0, c - window + 1) : 0;
      emit(P.dtc, s, 0, 1, kb, c + 1, kTcDecodeSplitKeys);
      continue;
    }
    if (q == 1 && g == 1) {
      const int kb = window > 0 ? std::max(0, c - window + 1) : 0;
      emit(P.decode, s, 0, 1, kb, c + 1, kDecodeSplitKeys);
      continue;
    }
    if (use_tc) {
      const int tpt = kTcUnitRows / g;
      for (int t0 = 0; t0 < q; t0 += tpt) {
        const int nt = std::min(tpt, q - t0);
        const int p0 = c + t0, p1 = c + t0 + nt - 1;
        const int kb = window > 0 ? std::max(0, p0 - window + 1) : 0;
        int split = nt * g <= 16 ? kTcDecodeSplitKeys : (1 << 30);
        const int nk = p1 + 1 - kb;
        const int pieces = dense_pieces.empty() ? 1 : dense_pieces[dense_next++];
        if (nt * g > 16 && pieces > 1)
          split = std::max(kTcMinSplitKeys, ((nk + pieces - 1) / pieces + 63) & ~63);
        emit(P.tc, s, t0, nt, kb, p1 + 1, split);
      }
      continue;
    }
    for (int t0 = 0; t0 < q; t0 += tok_per_tile) {
      const int nt = std::min(tok_per_tile, q - t0);
      const int p0 = c + t0, p1 = c + t0 + nt - 1;
      const int kb = window > 0 ? std::max(0, p0 - window + 1) : 0;
      emit(P.general, s, t0, nt, kb, p1 + 1, kSplitKeys);
    }
  }
  // longest units first (by 64-key stages), stable: a counting sort, so
  // planning stays linear in the number of units
  auto by_length = [&P](std::vector<WorkItem>& v) {
    if (v.size() < 2) return;
    constexpr int kBuckets = 4096;
    auto stages = [](const WorkItem& w) {
      const int n = (w.key_end - (w.key_begin - (w.key_begin & 63)) + 63) >> 6;
      return n < kBuckets - 1 ? n : kBuckets - 1;
    };
    std::vector<int32_t>& cnt = P.sort_count;
    cnt.assign(kBuckets + 1, 0);
    for (const WorkItem& w : v) ++cnt[kBuckets - 1 - stages(w)];
    int32_t run = 0;
    for (int b = 0; b <= kBuckets; ++b) {
      const int32_t c = cnt[b];
      cnt[b] = run;
      run += c;
    }
    P.sort_tmp.resize(v.size());
    for (const WorkItem& w : v) P.sort_tmp[cnt[kBuckets - 1 - stages(w)]++] = w;
    v.swap(P.sort_tmp);
  };
  // Query tiles: longest first by a coarse length (the top four bits of the
  // 64-key stage count: units within about 6 % of each other tie), and among
  // ties grouped by (kv head, first key, sequence). Units that read the same
  // keys of the same kv head then run at the same time on different SMs, so
  // their K/V tiles are fetched from DRAM about once and served from L2 to
  // the rest; ordered by exact length alone, the concurrent units of a long
  // prompt span every kv head and key range at once, more K/V than L2 holds.
  auto by_length_grouped = [](std::vector<WorkItem>& v) {
    auto coarse = [](const WorkItem& w) {
      int n = (w.key_end - (w.key_begin - (w.key_begin & 63)) + 63) >> 6;
      int sh = 0;
      while ((n >> sh) >= 16) ++sh;
      return (n >> sh) << sh;
    };
    std::stable_sort(v.begin(), v.end(), [&](const WorkItem& a, const WorkItem& b) {
      const int ca = coarse(a), cb = coarse(b);
      if (ca != cb) return ca > cb;
      if (a.kv_head != b.kv_head) return a.kv_head < b.kv_head;
      if (a.key_begin != b.key_begin) return a.key_begin < b.key_begin;
      return a.seq < b.seq;
    });
  };
  by_length(P.decode);
  by_length_grouped(P.tc);
  by_length(P.dtc);
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
