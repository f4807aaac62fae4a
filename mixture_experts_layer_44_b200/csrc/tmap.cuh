// Tensor maps (TMA descriptors) for bf16 tiles stored with the 128-byte
// swizzle, as the tensor-core kernels load them.
#pragma once

#include <cuda.h>

namespace moe_host {

// Encode the rank-2 or rank-3 bf16 tensor map of `base` with the given dims
// (innermost first), byte strides of the outer dims and box, 128-byte swizzle,
// zero fill outside the tensor.  Encoded maps are cached by (device, base,
// dims, strides, box).  Returns false if the driver entry point is missing
// or the layout is rejected.
bool encode_bf16_sw128(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                       const cuuint64_t* strides_bytes, const cuuint32_t* box);

// The same for an fp16 tensor (the target of TMA stores).
bool encode_f16_sw128(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                      const cuuint64_t* strides_bytes, const cuuint32_t* box);

// The same for an fp32 tensor (used as the target of TMA stores).
bool encode_f32_sw128(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                      const cuuint64_t* strides_bytes, const cuuint32_t* box);

}  // namespace moe_host
