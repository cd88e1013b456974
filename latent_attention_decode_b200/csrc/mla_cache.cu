// Appending decode tokens to the latent cache, with the RoPE key turned to its position here.
//
// Sources: "Ling-3.1-flash and the 7:1 hybrid: how much KV cache does a 560B model need at 1M
// tokens?", section "How big is the cache per token, exactly?" (a cached row is the 512-wide
// compressed latent followed by the 64-wide RoPE key, 576 bf16 values); "Ling-3.1-flash: a 560B
// hybrid-attention MoE, counted from its safetensors headers", section "Context: 1M in the
// claims, 262,144 in the config" (position enters only through RoPE on 64 of the 192 query-key
// dimensions of the MLA layers; rope_theta 6e6, no scaling).
//
// One CTA of 64 threads per new token: the latent row moves as 64 16-byte pieces; threads 0-31
// each turn one pair of the RoPE key, in fp64 (angle = position x inverse frequency, the
// frequencies computed on the host), and round each result to bf16 once.
//
// FP8 cache (the same page's "an FP8 cache would halve it"): every element x of that row (the RoPE
// key before its bf16 rounding) is stored as the E4M3 code of x / kv_scale, the quotient taken in
// fp32 (x rounded to fp32 first, exact for the bf16 latent) and rounded once to nearest even,
// saturating at +-448.
#include <cuda_bf16.h>

#include <cmath>

#include <type_traits>

#include "lad_common.cuh"
#include "sm100_ptx.cuh"

namespace {

constexpr int kDl = 512, kDr = 64, kDrow = kDl + kDr;

__device__ int g_cache_error = 0;

struct AppendArgs {
    const uint16_t *c_kv;   // [B][512]
    const uint16_t *k_pe;   // [B][64], not yet turned
    const int *positions;   // [B]
    void *cache;            // contiguous [B][Lmax][576] (block_table == nullptr) or a page pool
    long long seq_stride;   // contiguous: elements between sequences
    int Lmax;               // contiguous: rows per sequence
    const int *block_table; // paged: [B][bt_stride]
    int bt_stride, page_size, num_pages;
    int interleaved;
    float kv_scale;         // FP8 cache: a stored code is x / kv_scale
    double inv_freq[kDr / 2];
};

template <bool kFp8>
__global__ void __launch_bounds__(64) mla_cache_append_kernel(const __grid_constant__ AppendArgs a) {
    using Elem = typename std::conditional<kFp8, uint8_t, uint16_t>::type;
    const int b = blockIdx.x, t = threadIdx.x;
    const int pos = a.positions[b];
    Elem *dst = nullptr;
    Elem *const cache = static_cast<Elem *>(a.cache);
    if (a.block_table) {
        if (pos >= 0 && pos / a.page_size < a.bt_stride) {
            const int page = a.block_table[static_cast<long long>(b) * a.bt_stride + pos / a.page_size];
            if (page >= 0 && page < a.num_pages)
                dst = cache + (static_cast<long long>(page) * a.page_size + pos % a.page_size) * kDrow;
        }
    } else if (pos >= 0 && pos < a.Lmax) {
        dst = cache + static_cast<long long>(b) * a.seq_stride + static_cast<long long>(pos) * kDrow;
    }
    if (!dst) {
        if (t == 0) atomicCAS(&g_cache_error, 0, lad::kErrCacheAppend);
        return;
    }
    const uint4 lat = reinterpret_cast<const uint4 *>(a.c_kv + static_cast<size_t>(b) * kDl)[t];
    if constexpr (kFp8) {
        // 8 latent values -> 8 codes
        const uint32_t w[4] = {lat.x, lat.y, lat.z, lat.w};
        uint32_t c[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
            c[i] = lad::ptx::f32x2_to_e4m3x2(__fdiv_rn(lo, a.kv_scale), __fdiv_rn(hi, a.kv_scale));
        }
        reinterpret_cast<uint2 *>(dst)[t] = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
    } else {
        reinterpret_cast<uint4 *>(dst)[t] = lat;
    }
    if (t < kDr / 2) {
        const int ia = a.interleaved ? 2 * t : t, ib = a.interleaved ? 2 * t + 1 : t + kDr / 2;
        const uint16_t *k = a.k_pe + static_cast<size_t>(b) * kDr;
        const double x = static_cast<double>(lad::dev::bf16_to_f32(k[ia]));
        const double y = static_cast<double>(lad::dev::bf16_to_f32(k[ib]));
        double s, c;
        sincos(static_cast<double>(pos) * a.inv_freq[t], &s, &c);
        // separate roundings (no fused multiply-add), as a plain fp64 evaluation does
        const double u = __dsub_rn(__dmul_rn(x, c), __dmul_rn(y, s));
        const double w = __dadd_rn(__dmul_rn(y, c), __dmul_rn(x, s));
        if constexpr (kFp8) {
            const uint32_t c2 = lad::ptx::f32x2_to_e4m3x2(__fdiv_rn(__double2float_rn(u), a.kv_scale),
                                                          __fdiv_rn(__double2float_rn(w), a.kv_scale));
            dst[kDl + ia] = static_cast<uint8_t>(c2 & 0xff);
            dst[kDl + ib] = static_cast<uint8_t>(c2 >> 8);
        } else {
            dst[kDl + ia] = __bfloat16_as_ushort(__double2bfloat16(u));
            dst[kDl + ib] = __bfloat16_as_ushort(__double2bfloat16(w));
        }
    }
}

}  // namespace

namespace lad {
int take_device_error_cache(cudaStream_t s, int *code) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_cache_error, sizeof v, 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return set_error(LAD_ECUDA, "lad_device_error: %s", cudaGetErrorString(e));
    if (v) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_cache_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return set_error(LAD_ECUDA, "lad_device_error: %s", cudaGetErrorString(e));
    }
    *code = v;
    return LAD_OK;
}

void rope_inverse_frequencies(double theta, int d_rope, double *out) {
    for (int i = 0; i < d_rope / 2; ++i) out[i] = std::pow(theta, -2.0 * i / d_rope);
}
}  // namespace lad

namespace {
int append(const char *name, const lad_bf16 *c_kv, const lad_bf16 *k_pe, const int *positions, void *cache,
           long long cache_seq_stride, int Lmax, const int *block_table, int block_table_stride, int num_pages,
           int page_size, int B, int d_latent, int d_rope, float rope_theta, unsigned flags, bool fp8, float kv_scale,
           void *stream) {
    using lad::set_error;
    if (B < 0) return set_error(LAD_EINVAL, "%s: negative B", name);
    if (fp8 && (!(kv_scale > 0.f) || kv_scale == INFINITY))
        return set_error(LAD_EINVAL, "%s: kv_scale must be positive and finite", name);
    if (d_latent != kDl || d_rope != kDr) return set_error(LAD_EUNSUPPORTED, "%s: d_latent = 512, d_rope = 64 only", name);
    if (flags & ~LAD_FLAG_ROPE_INTERLEAVED) return set_error(LAD_EINVAL, "%s: unknown flags 0x%x", name, flags);
    if (!(rope_theta > 1.f) || rope_theta == INFINITY) return set_error(LAD_EINVAL, "%s: rope_theta must be > 1", name);
    if (B == 0) return LAD_OK;
    if (!c_kv || !k_pe || !positions || !cache) return set_error(LAD_EINVAL, "%s: null pointer", name);
    if (!lad::aligned(c_kv, 16) || !lad::aligned(cache, 16))
        return set_error(LAD_EUNSUPPORTED, "%s: c_kv and the cache must be 16-byte aligned", name);
    AppendArgs a{};
    a.c_kv = reinterpret_cast<const uint16_t *>(c_kv);
    a.k_pe = reinterpret_cast<const uint16_t *>(k_pe);
    a.positions = positions;
    a.cache = cache;
    a.interleaved = (flags & LAD_FLAG_ROPE_INTERLEAVED) ? 1 : 0;
    a.kv_scale = kv_scale;
    if (block_table) {
        if (page_size <= 0 || num_pages < 0 || block_table_stride < 0)
            return set_error(LAD_EINVAL, "%s: page_size > 0, num_pages and block_table_stride >= 0", name);
        a.block_table = block_table;
        a.bt_stride = block_table_stride;
        a.page_size = page_size;
        a.num_pages = num_pages;
    } else {
        const int mult = fp8 ? 16 : 8;  // rows stay 16-byte aligned
        if (Lmax < 0 || cache_seq_stride < static_cast<long long>(Lmax) * kDrow || cache_seq_stride % mult != 0)
            return set_error(LAD_EINVAL, "%s: cache_seq_stride must be >= Lmax*576 and a multiple of %d", name, mult);
        a.seq_stride = cache_seq_stride;
        a.Lmax = Lmax;
    }
    lad::rope_inverse_frequencies(static_cast<double>(rope_theta), kDr, a.inv_freq);
    if (fp8)
        mla_cache_append_kernel<true><<<B, 64, 0, lad::as_stream(stream)>>>(a);
    else
        mla_cache_append_kernel<false><<<B, 64, 0, lad::as_stream(stream)>>>(a);
    return lad::check_launch(name);
}
}  // namespace

extern "C" int mla_cache_append(const lad_bf16 *c_kv, const lad_bf16 *k_pe, const int *positions, lad_bf16 *cache,
                                long long cache_seq_stride, int Lmax, const int *block_table, int block_table_stride,
                                int num_pages, int page_size, int B, int d_latent, int d_rope, float rope_theta,
                                unsigned flags, void *stream) {
    return append("mla_cache_append", c_kv, k_pe, positions, cache, cache_seq_stride, Lmax, block_table,
                  block_table_stride, num_pages, page_size, B, d_latent, d_rope, rope_theta, flags, false, 1.f, stream);
}

extern "C" int mla_cache_append_fp8(const lad_bf16 *c_kv, const lad_bf16 *k_pe, const int *positions, uint8_t *cache,
                                    long long cache_seq_stride, int Lmax, const int *block_table,
                                    int block_table_stride, int num_pages, int page_size, int B, int d_latent,
                                    int d_rope, float rope_theta, float kv_scale, unsigned flags, void *stream) {
    return append("mla_cache_append_fp8", c_kv, k_pe, positions, cache, cache_seq_stride, Lmax, block_table,
                  block_table_stride, num_pages, page_size, B, d_latent, d_rope, rope_theta, flags, true, kv_scale,
                  stream);
}
