// Host-side helpers shared by the translation units of libispa: the
// thread-local error string, argument checks and TMA tensor-map encoding.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <string>

#include "ispa.h"

namespace ispa {

void set_last_error(const char* fmt, ...);

// Records `what` and returns ISPA_ERR_INVALID_ARG.
ispa_status_t invalid(const char* fmt, ...);
ispa_status_t unsupported(const char* fmt, ...);

// Checks the result of a kernel launch; ISPA_OK or ISPA_ERR_CUDA.
ispa_status_t check_launch(const char* kernel_name);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 2-D TMA map over a row-major [rows, inner] bf16 matrix with rows `row_bytes`
// apart; boxes of box_inner x box_rows elements, 128-byte swizzle, zero fill
// outside the matrix.
bool encode_map_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                        uint32_t box_inner, uint32_t box_rows);

// The same for a row-major [rows, inner] matrix of bytes (e4m3 codes).
bool encode_map_u8_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                      uint32_t box_inner, uint32_t box_rows);

// 2-D TMA map for output tiles of a row-major [rows, inner] matrix (fp32 or
// bf16): boxes of 32 x 32 elements, 128-byte swizzle for fp32 (one box row is
// 128 bytes), 64-byte swizzle for bf16.  Used by TMA stores and reductions.
bool encode_map_out_2d(CUtensorMap* map, const void* base, bool f32, uint64_t inner, uint64_t rows,
                       uint64_t row_bytes);

// Opt a kernel into `bytes` of dynamic shared memory (once per kernel/device).
ispa_status_t set_smem(const void* kernel, int bytes);

// Number of SMs of the current device.
int num_sms();

}  // namespace ispa
