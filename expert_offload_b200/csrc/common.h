// common.h - shared host helpers of libhfq4moe: status/message handling and
// argument checks.  Included by the .cpp and .cu translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cstdio>
#include <cstdarg>

#include "hfq4moe.h"

namespace hfq {

// Records a formatted message for hfq_last_error() and returns `st`.
hfq_status fail(hfq_status st, const char *fmt, ...);
// Clears the message (successful call).
hfq_status ok();

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t blocks_per_row(int cols) { return (size_t)(cols + HFQ4_BLOCK - 1) / HFQ4_BLOCK; }

inline size_t matrix_bytes(int rows, int cols)
{
    return (size_t)rows * blocks_per_row(cols) * HFQ4_BLOCK_BYTES;
}

inline size_t expert_bytes(int hidden, int inter)
{
    return 2 * matrix_bytes(inter, hidden) + matrix_bytes(hidden, inter);
}

// Shape checks shared by the forward entry points.
hfq_status check_shape(int hidden, int inter, int n_experts, int k);

}  // namespace hfq
