// Layout of the grouping plan of the grouped decode, shared by the host
// planner (host/group_plan.cpp) and the device kernels (kernels/*.cuh).
//
// Sequences forked from one parent hold the same physical blocks for their
// common prefix ["Your GPU was mostly empty", section "Paging's second gift:
// copy-on-write"]. The plan says which sequences of a decode batch read such a
// prefix together: a subgroup of up to members_per_subgroup(G) sequences and
// its shared prefix of c full blocks.
//
// Rule. A sequence whose context holds at least one full block, and whose
// first block-table entry is a valid block id, is keyed by that id; the batch
// is sorted by (key, sequence index) and every run of equal keys is cut, in
// that order, into subgroups of up to members_per_subgroup(G) members (a
// subgroup of one is dropped: its member is decoded alone). The shared prefix
// of a subgroup is its first c blocks, c = the number of leading block-table
// entries that are equal across all members, capped at every member's number
// of full blocks. Every member attends to all c * block_size shared tokens,
// and from block c on to its own.
//
// Plan (int32 words):
//   [0]             number of subgroups
//   [1]             most partitions of any subgroup's shared prefix
//   [2]             most partitions of any sequence's own range
//   [3]             shared blocks: the sum of c over subgroups
//   [4]             own blocks: the sum over sequences of the blocks from c on
//   [5, 8)          zero
//   [8, 8 + S)      per sequence: c of its subgroup, 0 for a sequence in none
//   [8 + S, ...)    per subgroup, kSubWords words:
//                   {c, number of members, 0, 0, member sequence indices}
// Partitions count partition_size tokens from the start of each range.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define KVP_HD __host__ __device__
#else
#define KVP_HD
#endif

namespace kvp {
namespace grp {

constexpr int kMaxSeqs = 4096;   // larger batches are decoded without grouping
constexpr int kMaxMembers = 16;  // columns of the tensor-core contraction
constexpr int kHdrWords = 8;
constexpr int kSubWords = 4 + kMaxMembers;

enum HeaderWord : int {
  kNumSub = 0,
  kSharedParts = 1,
  kOwnParts = 2,
  kSharedBlocks = 3,
  kOwnBlocks = 4,
};

KVP_HD constexpr int64_t sub_offset(int64_t S) { return kHdrWords + S; }
KVP_HD constexpr int64_t plan_words(int64_t S) { return kHdrWords + S + (S / 2 + 1) * kSubWords; }

// Columns of the contraction (8 for one query head per KV head, else 16)
// and the members of a subgroup that fill them (1 when grouping cannot help).
KVP_HD constexpr int plan_columns(int G) { return G == 1 ? 8 : 16; }
KVP_HD constexpr int members_per_subgroup(int G) {
  return G < 1 ? 1 : (plan_columns(G) / G < 1 ? 1 : plan_columns(G) / G);
}

}  // namespace grp
}  // namespace kvp
