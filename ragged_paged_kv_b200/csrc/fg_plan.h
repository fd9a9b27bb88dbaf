// Work planning for one ragged attention pass (host, integer work only).
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include "fg_internal.h"

namespace fg {

constexpr int kMaxGroup = 16;     // q heads per kv head served
constexpr int kGeneralRows = 16;  // query rows per general-path unit
constexpr int kSplitKeys = 1024;  // keys per split-KV partial (general path)
constexpr int kDecodeSplitKeys = 512;  // keys per unit of the MHA decode kernel
constexpr int kTcRows = 128;           // query rows per tensor-core tile
constexpr int kTcUnitRows = 256;       // query rows per tensor-core unit (two tiles sharing K/V)
constexpr int kTcDecodeSplitKeys = 2048;  // keys per unit for small (decode) tc tiles
constexpr int kDtcMaxGroup = 16;          // q heads per kv head the decode tc kernel serves
constexpr int kTcMinSplitKeys = 4096;     // shortest piece when a long query tile is split

struct Plan {
  std::vector<WorkItem> general;   // CUDA-core general path
  std::vector<WorkItem> decode;    // one-row MHA decode units (split-KV)
  std::vector<WorkItem> tc;        // tensor-core query tiles (prompt chunks)
  std::vector<WorkItem> dtc;       // one-token decodes on tensor cores (keys as MMA rows)
  std::vector<CombineItem> combine;
  std::vector<WorkItem> sort_tmp;  // scratch of the longest-first sort
  std::vector<int32_t> sort_count;
  std::vector<int32_t> sort_tmp_pieces;  // scratch: pieces per dense query tile
  int32_t part_rows = 0;         // partial rows the split units write
  int32_t max_combine_rows = 0;  // largest n_rows among combine items
  // packed device layout (bytes from the plan buffer's start)
  size_t off_general = 0, off_decode = 0, off_tc = 0, off_dtc = 0, off_combine = 0, total = 0;
  int32_t n_general = 0, n_decode = 0, n_tc = 0, n_dtc = 0, n_combine = 0;

  size_t bytes() const { return total; }
  void pack(void* dst) const;
};

// Cut the batch into work units: per sequence and kv head, tiles of new
// tokens, each over the key range its rows can see (causal, sliding window);
// long ranges are split into partials merged afterwards by the combine
// kernel. One-token queries with one q head per kv head go to the decode
// kernel in kDecodeSplitKeys-key units; everything else to the general path
// (up to kGeneralRows rows per unit, kSplitKeys keys per partial).
// use_tc: the tensor-core kernels may serve the batch (tensor maps built,
// g a power of two <= 128). Then one-token decodes with d = 128 and g <= 16
// go to the keys-as-rows decode kernel (dtc), other tokens to 128-row query
// tiles (tc); without it, MHA decodes go to the CUDA-core decode kernel and
// the rest to the general path.
// slots: CTAs the query-tile kernel runs with (for the long-tile split).
void build_plan(const std::vector<int32_t>& q_lens, const std::vector<int32_t>& ctx_lens,
                int n_kv_heads, int g, int head_dim, int window, bool use_tc, int slots, Plan* out);

}  // namespace fg
