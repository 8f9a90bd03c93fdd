// Where the keys of a decode sequence live.  Two layouts of the key cache:
//  * packed: sequence b's rows are cache rows cu[b] .. cu[b+1]-1 of a
//    [rows][H][d] tensor (cu_seqlens);
//  * paged: the cache is [pages][page_size][H][d] and key j of sequence b is
//    row j % page_size of page block_table[b][j / page_size]; seqlens[b]
//    rows are in use (page_size a power of two).
// Either way sequence b holds n_b context keys plus the g keys of the step
// (paper abstract: the decode group is one MTP step's queries).
#pragma once

#include <cstdint>

namespace pivot {

struct CacheIndex {
  const int32_t* cu;            // [B+1] packed layout, or null
  const int32_t* seqlens;       // [B] paged layout, or null
  const int32_t* block_table;   // [B][max_pages] (paged)
  int max_pages;
  int log2_page;

  __host__ __device__ bool decode() const { return cu != nullptr || seqlens != nullptr; }
  __device__ __forceinline__ int len(int b) const { return cu ? cu[b + 1] - cu[b] : seqlens[b]; }
  // cache row of key 0 in the packed layout (0 when paged)
  __device__ __forceinline__ long long row0(int b) const { return cu ? static_cast<long long>(cu[b]) : 0; }
  // cache row of key j of sequence b: r0 + j without a block table (the
  // packed layout, r0 = row0(b); prefill, r0 = 0), else through the table
  // (0 <= j < len(b) <= max_pages << log2_page)
  __device__ __forceinline__ long long row(int b, long long r0, int j) const {
    if (block_table == nullptr) return r0 + j;
    const int page = block_table[static_cast<long long>(b) * max_pages + (j >> log2_page)];
    return (static_cast<long long>(page) << log2_page) | (j & ((1 << log2_page) - 1));
  }
};

}  // namespace pivot
