// Layout of the split-KV decode plan (host-built, read by the decode kernels).
//
// The plan is one flat buffer:
//   PlanHeader
//   int32 cta_begin[num_ctas + 1]        work list c = items[cta_begin[c] .. cta_begin[c+1])
//   WorkItem items[num_items]            grouped by work list
//   CombineItem combine[num_combine]     (sequence, query) pairs split over several items
// Offsets are in bytes from the start of the plan and are multiples of 16.
#pragma once

#include <stdint.h>

namespace mla {

constexpr uint32_t kPlanMagic = 0x314C4D50u;  // "PML1"
constexpr int kPlanVersion = 1;

struct PlanHeader {
  uint32_t magic;
  int32_t version;
  int32_t batch, q_len, n_h;
  int32_t num_items, num_ctas, num_partials, num_combine;
  int32_t cta_off, items_off, combine_off;
  int32_t max_pages_used;  // largest page_end over all items
  int32_t reserved[3];
};
static_assert(sizeof(PlanHeader) == 64, "plan header is 64 bytes");

// One unit of work: query j of sequence b over logical pages [page_begin, page_end).
struct WorkItem {
  int32_t b;
  int32_t j;
  int32_t page_begin;
  int32_t page_end;
  int32_t slot;   // -1: the item covers the whole prefix and writes o/lse directly;
                  // >= 0: partial-result slot merged by the combine pass
  int32_t L;      // tokens in sequence b (including the new ones)
  int32_t qpos;   // absolute position of the query: L - q_len + j
  int32_t pad;
};
static_assert(sizeof(WorkItem) == 32, "work item is 32 bytes");

struct CombineItem {
  int32_t b, j, first_slot, n_parts;
};
static_assert(sizeof(CombineItem) == 16, "combine item is 16 bytes");

// Workspace layout for `num_partials` slots of n_h heads:
//   float o_part[num_partials][n_h][512]   (normalised partial latent outputs)
//   float lse_part[num_partials][n_h]      (natural-log sum-exp of each part)
inline size_t workspace_o_bytes(int num_partials, int n_h) {
  return (size_t)num_partials * n_h * 512 * sizeof(float);
}
inline size_t workspace_bytes(int num_partials, int n_h) {
  size_t o = workspace_o_bytes(num_partials, n_h);
  size_t l = ((size_t)num_partials * n_h * sizeof(float) + 255) & ~(size_t)255;
  return o + l;
}

}  // namespace mla
