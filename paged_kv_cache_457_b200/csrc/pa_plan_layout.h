// Layout of a cascade-decode plan (int32), shared by the host planner and the kernels:
//   [jobs: num_jobs x CJ_INTS][members: num_members][piece offsets: num_seqs + 1][piece rows: num_pieces]
// with the num_prefix_jobs prefix jobs first.
#pragma once

namespace pa {

constexpr int CJ_INTS = 8;     // ints per job
constexpr int CJ_SEQ = 0;      // sequence whose table row names the job's blocks
constexpr int CJ_T0 = 1;       // first 16-token tile
constexpr int CJ_T1 = 2;       // tile bound (exclusive); a suffix job also stops at its sequence's length
constexpr int CJ_MEMBERS = 3;  // first entry of the job's members in the member list
constexpr int CJ_NM = 4;       // members: sequences whose query heads are the job's columns
constexpr int CJ_ROW = 5;      // first partial row of the job (per kv head); split s, member i, head j ->
                               // row + (s * members + i) * G + j
constexpr int CJ_KIND = 6;     // CJ_PREFIX or CJ_SUFFIX
constexpr int CJ_SPLIT = 7;    // prefix job: its tiles are dealt round-robin to `split` warp sets (1, 2 or 4), each
                               // leaving its own partial rows; suffix job: 1
constexpr int CJ_PREFIX = 0, CJ_SUFFIX = 1;
constexpr int CASCADE_CONSUMERS = 4;  // warps per block of the partial kernel: a prefix job's row tiles (16
                                      // member x head rows each) times its split, or one suffix job each
constexpr int CASCADE_TILE = 16;      // tokens per tile
constexpr int CASCADE_DEFAULT_CHUNK_TOKENS = 320;  // measured on 8 groups x 8 sequences sharing 1024 tokens, 32 q / 8 kv
                                                   // heads: 128, 192, 256, 320, 384, 512 gave 43.0, 44.4, 43.1, 39.0,
                                                   // 41.0, 45.1 us per step

}  // namespace pa
