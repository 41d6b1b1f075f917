// Internal helpers shared by the library's translation units.
#pragma once

#include <cstdarg>
#include <cstddef>
#include <cstdint>

#include "tq.h"

namespace tq {

// Records a printf-style message as this thread's last error and returns `st`.
tq_status fail(tq_status st, const char* fmt, ...);
void clear_error();

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline int64_t idx_row_bytes(int d, int bits) { return static_cast<int64_t>(d) * bits / 8; }
inline int64_t sign_words(int d) { return (d + 31) / 32; }

// Validates d / bits of a layout; returns TQ_OK or an error with a message.
tq_status check_layout(const tq_layout* layout);
tq_status check_bits(int bits, const char* what);

constexpr int kMaxD = 256;

// Counts kernel launches issued by the library (tq_kernel_launches).
void count_launch(int n = 1);

// Limit of the tcgen05 kernels' pipeline waits, in ns: 2 s, or the value of
// the environment variable TQ_TEST_WAIT_NS (tests shorten it to make the waits
// run out). The waits that drain copies and MMAs before exit keep 2 s.
uint64_t pipeline_wait_ns();

}  // namespace tq
