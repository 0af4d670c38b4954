// stepq_internal.h -- host-side helpers shared by the libstepq translation units.
#pragma once

#include <cstdint>
#include <cstdio>
#include <cstring>
#include <string>

#include "stepq.h"

namespace stepq {

// Records the message of the last error of the calling thread; returns `code`.
int set_error(int code, const char* fmt, ...);
void clear_error();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool dims_supported(const stepq_dims& d) {
    return (d.dk == 64 || d.dk == 128) && d.dv == d.dk;
}

// Common validation of the tile dimensions; returns STEPQ_OK or an error code.
inline int check_dims(const stepq_dims& d, const char* fn) {
    if (d.B < 0 || d.H <= 0) return set_error(STEPQ_EINVAL, "%s: B=%d H=%d", fn, d.B, d.H);
    if (!dims_supported(d))
        return set_error(STEPQ_EUNSUPPORTED, "%s: dk=%d dv=%d (need dk == dv in {64, 128})", fn, d.dk, d.dv);
    if (d.gate_per_channel != 0 && d.gate_per_channel != 1)
        return set_error(STEPQ_EINVAL, "%s: gate_per_channel=%d", fn, d.gate_per_channel);
    return STEPQ_OK;
}

// Validates that each pointer is non-null and 16-byte aligned.
int check_ptrs(const char* fn, std::initializer_list<std::pair<const char*, const void*>> ptrs);

// Maps a CUDA launch status to STEPQ_OK / STEPQ_ECUDA (with the message recorded).
int check_launch(const char* fn);

// Device address of the current device's error word (the one stepq_read_device_flags reads).
int device_flags_ptr(uint32_t** p);

// Grid of a persistent kernel on the current device: the SM count times the CTAs of `threads`
// threads and `smem` bytes of dynamic shared memory that fit on one SM, capped at `tiles`. The
// kernel's shared-memory attribute and the occupancy are set up once per (kernel, device).
int persistent_grid(const void* kernel, int threads, size_t smem, long long tiles, const char* fn, int* grid);

}  // namespace stepq
