// Layout of the packed plan of the packed grouped decode, shared by the host
// planner (host/group_plan.cpp) and the device kernels.
//
// Sequences forked from one parent hold the same physical blocks for their
// common prefix ["Your GPU was mostly empty", section "Paging's second gift:
// copy-on-write"]. The packed decode reads every block of a batch once per
// group of the sequences that hold it, with one tensor-core kernel: each
// group's blocks form one stream - the shared prefix (every member attends to
// it), then each member's own blocks (only that member attends) - cut into
// chunks of a fixed number of blocks. A chunk is a unit of the kernel, whose
// columns are the members' query heads: a column takes a token's score only
// where the token's block is its member's (a per-block column mask), so one
// key tile may hold blocks of several members.
//
// Groups: the grouping rule of group_layout.h (sequences keyed by their first
// block, runs cut into subgroups of at most members_per_subgroup(G), shared
// prefix = the leading table entries equal across the members, capped at full
// blocks); every other sequence is a group of one with no shared prefix.
//
// Plan (int32 words):
//   [0] groups            [1] units per KV head       [2] entries
//   [3] most chunks of any group (partial slots per sequence and head)
//   [4] block size        [5] blocks per chunk
//   [6] word offset of the unit table   [7] word offset of the entries
//   [8, 8 + S)            per sequence: its group
//   per group, kGroupWords words:
//       {first entry, members, entries, chunks, member sequences [16]}
//   per unit, kUnitWords words (longest first):
//       {group, first entry, entries (<= blocks per chunk), chunk index}
//   per entry, 2 words: {block id, column mask << 8 | valid tokens of the block}
// Column j of a group is query head g * G + j % G of member j / G.
#pragma once

#include <stdint.h>

#include "group_layout.h"

namespace kvp {
namespace pack {

constexpr int kHdrWords = 8;
constexpr int kGroupWords = 4 + grp::kMaxMembers;
constexpr int kUnitWords = 4;

enum HeaderWord : int {
  kGroups = 0,
  kUnits = 1,
  kEntries = 2,
  kMaxChunks = 3,
  kBlockSize = 4,
  kChunkBlocks = 5,
  kUnitOffset = 6,
  kEntryOffset = 7,
};

KVP_HD constexpr int64_t group_offset(int64_t S) { return kHdrWords + S; }

// Words a plan of S sequences with at most MB blocks each can need: every
// sequence a group of its own, every block an entry, every entry a unit.
KVP_HD constexpr int64_t plan_words_bound(int64_t S, int64_t MB) {
  return kHdrWords + S + S * kGroupWords + S * MB * (kUnitWords + 2);
}

}  // namespace pack
}  // namespace kvp
