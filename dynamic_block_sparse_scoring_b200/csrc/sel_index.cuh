// Device buffers of the selected-block inverted index (see sel_index.cu).
#pragma once

#include <stdint.h>

#include <algorithm>

#include "common.cuh"

namespace nsa {

struct SelIndex {
    int32_t* cnt;       // [L] pairs per list, L = B * Hsel * nb_all
    int32_t* off;       // [L + 1] list offsets (exclusive scan); off[L] = pairs
    int32_t* item_off;  // [L + 1] first work item of each list; item_off[L] = items
    int32_t* cursor;    // [L] fill cursors
    int32_t* list;      // [pairs] query * SEL_SLOTS + slot, grouped by list
    int4* items;        // [items] (list id, first pair, pair count, 0)
};

// Lists are keyed by (query chunk, selection unit, block): list id =
// (chunk * B * Hsel + b * Hsel + u) * nb_all + block, chunk = query / SEL_CHUNK.
// Work items are therefore ordered chunk by chunk.  Longer chunks give longer
// lists (fuller 128-row work items, fewer K/V block loads) at the price of a
// query working set larger than L2; on the 64k prefill 8192 measured best
// (block-major kernel 8.0 ms against 8.4 at 2048, 9.4 at 1024, 7.9 at one
// chunk whose index build costs 0.3 ms more).
constexpr int SEL_CHUNK = 8192;
// A list entry is query * SEL_SLOTS + slot: up to 64 kept (sub-)blocks per query
// row, queries below 2^25.
constexpr int SEL_SLOT_BITS = 6;
constexpr int SEL_SLOTS = 1 << SEL_SLOT_BITS;
__host__ __device__ __forceinline__ int pair_query(int e) { return e >> SEL_SLOT_BITS; }
__host__ __device__ __forceinline__ int pair_slot(int e) { return e & (SEL_SLOTS - 1); }
inline int sel_chunks(const Shape& s) { return (s.Tq + SEL_CHUNK - 1) / SEL_CHUNK; }
inline size_t sel_lists_per_chunk(const Shape& s) { return (size_t)s.B * s.Hsel * s.nb_all; }

// Upper bounds used to size the workspace.
inline size_t sel_pairs_max(const Shape& s) { return (size_t)s.B * s.Hsel * s.Tq * s.topk; }
// rows of the selected-branch partial buffers: one per (pair, head of the unit)
inline size_t sel_partial_rows(const Shape& s) { return sel_pairs_max(s) * s.heads_per_unit; }
inline size_t sel_lists(const Shape& s) { return (size_t)sel_chunks(s) * sel_lists_per_chunk(s); }
// (+32 / +64 slack entries: the block-major producer reads 32 items / 64 list
// entries at a time past the last valid one)
inline size_t sel_items_max(const Shape& s, int tok) {
    return sel_pairs_max(s) / tok + sel_lists(s) + 1 + 32;
}
inline size_t sel_list_alloc(const Shape& s) { return sel_pairs_max(s) + 64; }

cudaError_t launch_sel_index(const Shape& s, const int32_t* idx, const SelIndex& x, int tok,
                             cudaStream_t st);

}  // namespace nsa
