// Host-side helpers shared by the launchers: tensor-map encoding, the
// per-device status word and small validation utilities.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/attn_b200.h"

namespace ea {

// Device address of this device's status word (created on first use).
// Returns nullptr if CUDA fails.
int* device_status_ptr();

// Encode a 4-D bf16 tile map with 128-byte swizzle.
//   dims    innermost first (elements)
//   strides byte strides of dims 1..3
//   box     tile extent per dim (box[0] * 2 bytes must be <= 128)
// Returns false if the driver rejects the description.
bool encode_bf16_4d(CUtensorMap* map, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                    const uint32_t box[4]);

// The same for 8-bit elements (box[0] must be <= 128).
bool encode_u8_4d(CUtensorMap* map, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                  const uint32_t box[4]);

// The same for fp32 elements (box[0] * 4 bytes must be <= 128).
bool encode_f32_4d(CUtensorMap* map, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                   const uint32_t box[4]);

// Encode a 2-D bf16 tile map with 128-byte swizzle (stride of dim 1).
bool encode_bf16_2d(CUtensorMap* map, const void* base, const uint64_t dims[2], const uint64_t strides[1],
                    const uint32_t box[2]);

// Encode a 3-D bf16 tile map with 128-byte swizzle (strides of dims 1..2).
bool encode_bf16_3d(CUtensorMap* map, const void* base, const uint64_t dims[3], const uint64_t strides[2],
                    const uint32_t box[3]);

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Raise the dynamic shared-memory limit of a kernel once per device.
int ensure_smem_attr(const void* kernel, int bytes, int* done_mask);

// Streaming multiprocessors of the current device, or of device `dev`
// (0 if the device does not exist or CUDA fails).
int current_sm_count();
int sm_count_of(int dev);

}  // namespace ea
