// Host side of cascade decode: grouping a batch by shared leading blocks, and the work plan that
// pa_decode_cascade runs ("4. vLLM核心机制" section 4.2: the blocks of a shared prefix are named by several
// block tables; reading them once per group instead of once per sequence is what the sharing saves).
// Plain C++ (no CUDA): it runs on the host and is tested without a GPU.
#include <algorithm>
#include <cstdint>
#include <map>
#include <vector>

#include "pa_b200.h"
#include "pa_plan_layout.h"

namespace {

bool supported_block_size(int32_t bs) { return bs == 16 || bs == 32; }

}  // namespace

extern "C" {

int pa_find_prefix_groups(const int32_t *block_tables, const int32_t *context_lens, int32_t num_seqs,
                          int32_t block_table_stride, int32_t block_size, int32_t min_prefix_blocks,
                          int32_t *group_offsets, int32_t *group_members, int32_t *group_prefix_blocks,
                          int32_t *num_groups) {
  if (num_seqs < 0 || block_table_stride <= 0) return PA_ERR_SHAPE;
  if (!supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
  if (!group_offsets || !num_groups || (num_seqs > 0 && (!block_tables || !context_lens || !group_members ||
                                                         !group_prefix_blocks)))
    return PA_ERR_NULL;
  const int64_t cap = (int64_t)block_table_stride * block_size;
  for (int32_t s = 0; s < num_seqs; ++s)
    if (context_lens[s] < 0 || context_lens[s] > cap) return PA_ERR_SHAPE;
  const int32_t min_blocks = std::max(1, min_prefix_blocks);
  // candidate groups: sequences with at least one full block, keyed by their first block (members in order)
  std::map<int32_t, std::vector<int32_t>> by_first;
  std::vector<int32_t> first_member_order;
  for (int32_t s = 0; s < num_seqs; ++s) {
    if (context_lens[s] / block_size < 1) continue;
    const int32_t b0 = block_tables[(int64_t)s * block_table_stride];
    auto &v = by_first[b0];
    if (v.empty()) first_member_order.push_back(b0);
    v.push_back(s);
  }
  int32_t ng = 0, nmem = 0;
  group_offsets[0] = 0;
  for (int32_t key : first_member_order) {  // in order of each candidate's first member
    const std::vector<int32_t> &mem = by_first[key];
    if (mem.size() < 2) continue;
    int32_t P = block_table_stride;
    for (int32_t m : mem) P = std::min(P, context_lens[m] / block_size);  // full blocks only
    const int32_t *lead = block_tables + (int64_t)mem[0] * block_table_stride;
    for (int32_t j = 0; j < P; ++j) {
      bool same = true;
      for (size_t i = 1; i < mem.size() && same; ++i) same = block_tables[(int64_t)mem[i] * block_table_stride + j] == lead[j];
      if (!same) {
        P = j;
        break;
      }
    }
    if (P < min_blocks) continue;
    for (int32_t m : mem) group_members[nmem++] = m;
    group_prefix_blocks[ng] = P;
    group_offsets[++ng] = nmem;
  }
  *num_groups = ng;
  return PA_OK;
}

int pa_cascade_plan(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t block_size,
                    int32_t max_context_len, int32_t chunk_tokens, int32_t num_groups, const int32_t *group_offsets,
                    const int32_t *group_members, const int32_t *group_prefix_blocks, int32_t *plan,
                    int64_t plan_capacity, pa_cascade_info *info) {
  if (!info) return PA_ERR_NULL;
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_context_len < 0 || num_groups < 0 ||
      plan_capacity < 0)
    return PA_ERR_SHAPE;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_HEADS;
  const int32_t G = num_q_heads / num_kv_heads;
  if (G > 8 || !supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
  if (chunk_tokens < 0 || chunk_tokens % pa::CASCADE_TILE != 0) return PA_ERR_PARTITION;
  const int32_t CH = (chunk_tokens == 0 ? pa::CASCADE_DEFAULT_CHUNK_TOKENS : chunk_tokens) / pa::CASCADE_TILE;
  if (num_groups > 0 && (!group_offsets || !group_prefix_blocks)) return PA_ERR_NULL;
  if (num_groups > 0 && group_offsets[0] != 0) return PA_ERR_SHAPE;
  for (int32_t g = 0; g < num_groups; ++g)
    if (group_offsets[g + 1] <= group_offsets[g] || group_prefix_blocks[g] < 0 ||
        (int64_t)group_prefix_blocks[g] * block_size > max_context_len)
      return PA_ERR_SHAPE;
  const int32_t total_members = num_groups > 0 ? group_offsets[num_groups] : 0;
  if (total_members > 0 && !group_members) return PA_ERR_NULL;
  std::vector<int32_t> prefix_tiles(num_seqs, 0);  // shared tiles of each sequence's group (0: none)
  std::vector<char> seen(num_seqs, 0);
  for (int32_t g = 0; g < num_groups; ++g)
    for (int32_t i = group_offsets[g]; i < group_offsets[g + 1]; ++i) {
      const int32_t m = group_members[i];
      if (m < 0 || m >= num_seqs || seen[m]) return PA_ERR_SHAPE;  // every sequence in at most one group
      seen[m] = 1;
      prefix_tiles[m] = group_prefix_blocks[g] * (block_size / pa::CASCADE_TILE);
    }

  const int32_t max_tiles = (max_context_len + pa::CASCADE_TILE - 1) / pa::CASCADE_TILE;
  // a prefix job's members fill up to CASCADE_CONSUMERS row tiles of 16 (member, head) rows; a job with fewer
  // row tiles deals its tiles to `split` sets of warps so that every warp of the block works
  const int32_t per_tile = 16 / G;
  const int32_t per_job = pa::CASCADE_CONSUMERS * per_tile;
  std::vector<int32_t> jobs, members;
  std::vector<std::vector<int32_t>> pieces(num_seqs);  // partial rows of each sequence, in merge order
  int64_t rows = 0;
  auto add_job = [&](int32_t seq, int32_t t0, int32_t t1, int32_t mfirst, int32_t nm, int32_t kind, int32_t split) {
    const int32_t job[pa::CJ_INTS] = {seq, t0, t1, mfirst, nm, (int32_t)rows, kind, split};
    static_assert(pa::CJ_SEQ == 0 && pa::CJ_T0 == 1 && pa::CJ_T1 == 2 && pa::CJ_MEMBERS == 3 && pa::CJ_NM == 4 &&
                      pa::CJ_ROW == 5 && pa::CJ_KIND == 6 && pa::CJ_SPLIT == 7 && pa::CJ_INTS == 8,
                  "job fields in the order written here");
    jobs.insert(jobs.end(), job, job + pa::CJ_INTS);
    rows += (int64_t)nm * G * split;
  };
  // prefix jobs first (the long ones start early): per group, per column set, per chunk of the shared tiles
  for (int32_t g = 0; g < num_groups; ++g) {
    const int32_t PT = group_prefix_blocks[g] * (block_size / pa::CASCADE_TILE);
    const int32_t n = group_offsets[g + 1] - group_offsets[g];
    if (PT == 0) continue;
    const int32_t mlist = (int32_t)members.size();
    members.insert(members.end(), group_members + group_offsets[g], group_members + group_offsets[g + 1]);
    const int32_t lead = group_members[group_offsets[g]];
    for (int32_t c0 = 0; c0 < n; c0 += per_job) {
      const int32_t nm = std::min(per_job, n - c0);
      const int32_t n_rt = (nm + per_tile - 1) / per_tile;
      const int32_t split = n_rt == 1 ? 4 : n_rt == 2 ? 2 : 1;
      for (int32_t t0 = 0; t0 < PT; t0 += CH) {
        const int64_t row = rows;
        add_job(lead, t0, std::min(PT, t0 + CH), mlist + c0, nm, pa::CJ_PREFIX, split);
        for (int32_t sp = 0; sp < split; ++sp)
          for (int32_t i = 0; i < nm; ++i)
            pieces[members[mlist + c0 + i]].push_back((int32_t)(row + ((int64_t)sp * nm + i) * G));
      }
    }
  }
  const int32_t num_prefix_jobs = (int32_t)(jobs.size() / pa::CJ_INTS);
  // suffix jobs: per sequence, per chunk of its own tiles up to the call's bound
  const int32_t self = (int32_t)members.size();
  for (int32_t s = 0; s < num_seqs; ++s) members.push_back(s);
  for (int32_t s = 0; s < num_seqs; ++s)
    for (int32_t t0 = prefix_tiles[s]; t0 < max_tiles; t0 += CH) {
      pieces[s].push_back((int32_t)rows);
      add_job(s, t0, std::min(max_tiles, t0 + CH), self + s, 1, pa::CJ_SUFFIX, 1);
    }
  if (rows > INT32_MAX / 2) return PA_ERR_SHAPE;

  int64_t num_pieces = 0;
  for (const auto &p : pieces) num_pieces += (int64_t)p.size();
  info->num_seqs = num_seqs;
  info->num_q_heads = num_q_heads;
  info->num_kv_heads = num_kv_heads;
  info->block_size = block_size;
  info->max_context_len = max_context_len;
  info->num_jobs = (int32_t)(jobs.size() / pa::CJ_INTS);
  info->num_prefix_jobs = num_prefix_jobs;
  info->num_members = (int32_t)members.size();
  info->num_pieces = (int32_t)num_pieces;
  info->rows_per_head = (int32_t)rows;
  info->plan_ints = (int64_t)jobs.size() + (int64_t)members.size() + (num_seqs + 1) + num_pieces;
  if (!plan) return PA_OK;
  if (plan_capacity < info->plan_ints) return PA_ERR_WORKSPACE;
  int32_t *p = plan;
  p = std::copy(jobs.begin(), jobs.end(), p);
  p = std::copy(members.begin(), members.end(), p);
  int32_t off = 0;
  for (int32_t s = 0; s < num_seqs; ++s) {
    *p++ = off;
    off += (int32_t)pieces[s].size();
  }
  *p++ = off;
  for (const auto &ps : pieces) p = std::copy(ps.begin(), ps.end(), p);
  return PA_OK;
}

}  // extern "C"
