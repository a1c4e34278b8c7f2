// Host-side helpers shared by the library's translation units.
#pragma once

#include <cstdarg>
#include <cstddef>
#include <cstdint>
#include <string>

#include "pkv.h"

namespace pkv {

// Record a printf-style message as this thread's last error and return `code`.
int set_error(int code, const char* fmt, ...);
void clear_error();

// The checks of a decode call that need no pointer (sizes, output type, path, partition), shared
// by the decode entry points (decode.cu).  PKV_OK and the partition to use, or the error code.
int decode_check_sizes(int out_dtype, bool kv8, int max_blocks_per_seq, int max_context_len, int num_seqs,
                       int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                       int partition_tokens, int path, int* partition_out);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace pkv
