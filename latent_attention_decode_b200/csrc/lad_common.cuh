// Shared host/device helpers of the decode library: error recording, bf16 conversion, argument
// checks, and the bounded-wait primitive every on-chip barrier wait goes through.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "lad.h"

namespace lad {

// Records a message for lad_last_error() on the calling thread and returns `code`.
int set_error(int code, const char *fmt, ...);

// Turns the last CUDA launch error into LAD_ECUDA (with the CUDA message) or LAD_OK.
int check_launch(const char *what);

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// Streaming-multiprocessor count of the current device (cached per device).
int device_sm_count();

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no libcuda link).
// Returned untyped; the caller casts it to the driver signature from <cuda.h>.
void *tensor_map_encoder_raw();

// Tags stored in the device error word when a bounded wait gives up (and one input check).
enum DeviceErrorTag : int {
    kErrNone = 0,
    kErrMlaProducer = 0x101,
    kErrMlaMma = 0x102,
    kErrMlaSoftmax = 0x103,
    kErrMlaEpilogue = 0x104,
    kErrMlaBlockTable = 0x105,  // a paged call met a block-table entry outside the pool (not a wait)
    kErrMlaQRange = 0x106,      // FP8-cache call: a query value beyond the f16 range (not a wait)
    kErrMlaConvert = 0x107,     // FP8-cache call: the widening warps gave up a wait
    kErrCacheAppend = 0x301,    // mla_cache_append: a position with no row to write (not a wait)
    kErrPrefill = 0x201,
    kErrKdaPair = 0x501,        // KDA decode, two heads per CTA: the second head's state copy never landed
};

// Host-side readers of the per-module device error words (each clears its word).
int take_device_error_mla(cudaStream_t s, int *code);
int take_device_error_prefill(cudaStream_t s, int *code);
int take_device_error_cache(cudaStream_t s, int *code);
int take_device_error_kda(cudaStream_t s, int *code);

// pow(theta, -2i/d) for the d/2 RoPE pairs, on the host (the oracle computes them the same way)
void rope_inverse_frequencies(double theta, int d_rope, double *out);

}  // namespace lad

// ---------------------------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------------------------
namespace lad::dev {

__device__ __forceinline__ float bf16_to_f32(uint16_t bits) {
    return __uint_as_float(static_cast<uint32_t>(bits) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// Two bf16 packed in a 32-bit word, low half first in memory.
__device__ __forceinline__ float2 bf16x2_to_f32(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
    return static_cast<uint32_t>(f32_to_bf16(lo)) | (static_cast<uint32_t>(f32_to_bf16(hi)) << 16);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Upper bound of any single wait on an on-chip barrier. Far above every legitimate wait (the
// longest is one tile's HBM fetch behind a full GPU), short enough to give the GPU back fast.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

}  // namespace lad::dev
