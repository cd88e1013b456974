// KDA short convolution: one decode step of the width-4 causal depthwise convolution that q, k
// and v pass through, with the tail (last K-1 inputs per channel) shifted in place.
//
// Source: "Ling-3.1-flash: a 560B hybrid-attention MoE, counted from its safetensors headers",
// sections "How KDA and MLA split the work" (short causal convolution of width 4) and "Does
// 292 GiB fit on four Hopper GPUs?" (the kept convolution tails).
//
// Elementwise over (sequence, channel): a thread takes 8 adjacent channels (16-byte vectors)
// so every load and store is a coalesced 128-bit access. Per channel it reads x, three tail
// values and four taps and writes y and the three shifted tail values: HBM-bound, with the taps
// ([Cch][4], 196 KiB at the pages' shape) shared by all sequences through L2.
#include "lad_common.cuh"

namespace {

using lad::dev::bf16x2_to_f32;
using lad::dev::f32x2_to_bf16x2;

constexpr int kTaps = 4;
constexpr int kThreads = 256;

struct Vec8 {
    float v[8];
};

__device__ __forceinline__ Vec8 unpack8(const uint4 &w) {
    Vec8 r;
    float2 a = bf16x2_to_f32(w.x), b = bf16x2_to_f32(w.y), c = bf16x2_to_f32(w.z), d = bf16x2_to_f32(w.w);
    r.v[0] = a.x; r.v[1] = a.y; r.v[2] = b.x; r.v[3] = b.y;
    r.v[4] = c.x; r.v[5] = c.y; r.v[6] = d.x; r.v[7] = d.y;
    return r;
}

__device__ __forceinline__ uint4 pack8(const Vec8 &r) {
    return make_uint4(f32x2_to_bf16x2(r.v[0], r.v[1]), f32x2_to_bf16x2(r.v[2], r.v[3]),
                      f32x2_to_bf16x2(r.v[4], r.v[5]), f32x2_to_bf16x2(r.v[6], r.v[7]));
}

__global__ void __launch_bounds__(kThreads)
kda_conv_kernel(const uint4 *__restrict__ x, uint4 *__restrict__ tail, const uint4 *__restrict__ w,
                const uint4 *__restrict__ bias, uint4 *__restrict__ y, long long n_vec, int c8, int silu) {
    const long long idx = static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x;
    if (idx >= n_vec) return;
    const long long b = idx / c8;
    const int cv = static_cast<int>(idx - b * c8);

    const uint4 xr = __ldcs(x + idx);
    uint4 *tb = tail + b * (kTaps - 1) * c8 + cv;
    const uint4 t0r = __ldcs(tb), t1r = __ldcs(tb + c8), t2r = __ldcs(tb + 2 * c8);
    // taps of 8 channels: 8 x 4 bf16 = 4 vectors, channel j's taps at positions 4j..4j+3
    const uint4 *wp = w + static_cast<size_t>(cv) * kTaps;
    const Vec8 w01 = unpack8(__ldg(wp + 0)), w23 = unpack8(__ldg(wp + 1));
    const Vec8 w45 = unpack8(__ldg(wp + 2)), w67 = unpack8(__ldg(wp + 3));
    const Vec8 xs = unpack8(xr), t0 = unpack8(t0r), t1 = unpack8(t1r), t2 = unpack8(t2r);
    Vec8 bs;
    if (bias) {
        bs = unpack8(__ldg(bias + cv));
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) bs.v[j] = 0.f;
    }

    Vec8 out;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const Vec8 &wv = (j < 2) ? w01 : (j < 4) ? w23 : (j < 6) ? w45 : w67;
        const int o = (j & 1) * 4;
        float acc = wv.v[o + 0] * t0.v[j];
        acc = fmaf(wv.v[o + 1], t1.v[j], acc);
        acc = fmaf(wv.v[o + 2], t2.v[j], acc);
        acc = fmaf(wv.v[o + 3], xs.v[j], acc);
        acc += bs.v[j];
        if (silu) acc = acc / (1.f + expf(-acc));
        out.v[j] = acc;
    }
    __stcs(y + idx, pack8(out));
    __stcs(tb, t1r);
    __stcs(tb + c8, t2r);
    __stcs(tb + 2 * c8, xr);
}

}  // namespace

extern "C" int kda_conv_update(const lad_bf16 *x, lad_bf16 *conv_tail, const lad_bf16 *w, const lad_bf16 *bias,
                               lad_bf16 *y, int B, int Cch, int K, unsigned flags, void *stream) {
    using lad::set_error;
    if (B < 0 || Cch < 0) return set_error(LAD_EINVAL, "kda_conv_update: negative B or Cch");
    if (K != kTaps) return set_error(LAD_EUNSUPPORTED, "kda_conv_update: K = 4 only");
    if (Cch % 8 != 0) return set_error(LAD_EUNSUPPORTED, "kda_conv_update: Cch must be a multiple of 8");
    if (flags & ~LAD_FLAG_SILU) return set_error(LAD_EINVAL, "kda_conv_update: unknown flags 0x%x", flags);
    if (B == 0 || Cch == 0) return LAD_OK;
    if (!x || !conv_tail || !w || !y) return set_error(LAD_EINVAL, "kda_conv_update: null pointer");
    if (!lad::aligned(x, 16) || !lad::aligned(conv_tail, 16) || !lad::aligned(w, 16) || !lad::aligned(y, 16) ||
        (bias && !lad::aligned(bias, 16)))
        return set_error(LAD_EUNSUPPORTED, "kda_conv_update: pointers must be 16-byte aligned");
    if (y == x || y == conv_tail) return set_error(LAD_EINVAL, "kda_conv_update: y aliases an input");
    const int c8 = Cch / 8;
    const long long n_vec = static_cast<long long>(B) * c8;
    const long long blocks = (n_vec + kThreads - 1) / kThreads;
    if (blocks > 0x7fffffffLL) return set_error(LAD_EUNSUPPORTED, "kda_conv_update: too large");
    kda_conv_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, lad::as_stream(stream)>>>(
        reinterpret_cast<const uint4 *>(x), reinterpret_cast<uint4 *>(conv_tail), reinterpret_cast<const uint4 *>(w),
        reinterpret_cast<const uint4 *>(bias), reinterpret_cast<uint4 *>(y), n_vec, c8,
        (flags & LAD_FLAG_SILU) ? 1 : 0);
    return lad::check_launch("kda_conv_update");
}
