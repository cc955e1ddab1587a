// Host-side helpers shared by the C-ABI entry points: error reporting and
// argument validation.  No device code here.
#pragma once

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <string>

#include "../../include/tq.h"

namespace tq {

// Set the thread-local error message and return `code`.
int set_error(int code, const char* fmt, ...);
// Clear the message (successful call).
void clear_error();

inline bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// kb = number of Lloyd-Max index bits for a parameter set.
inline int index_bits(const tq_params* p) { return p->mode == TQ_MODE_PROD ? p->bits - 1 : p->bits; }

// Validate a tq_params struct; returns TQ_OK or a TQ_E* (message set).
int check_params(const tq_params* p, const char* who);
// TQ_EUNSUPPORTED unless the codes are in the canonical bit-plane layout.
int check_planes(const tq_params* p, const char* who);

}  // namespace tq
