// KDA decode: one token of the gated delta rule per (sequence, head), streaming the fp32 state
// once through registers.
//
// Source: "Ling-3.1-flash: a 560B hybrid-attention MoE, counted from its safetensors headers",
// section "How KDA and MLA split the work" (128x128 state per head, per-channel decay alpha,
// per-head write strength beta, gated delta rule); "Ling-3.1-flash and the 7:1 hybrid...",
// section "Why would a model keep only 9 full-attention layers?" (Gated DeltaNet lineage).
//
// Per (b, h), with S of shape [d_k rows][d_v columns]:
//   S' = Diag(alpha) S;  u = beta (v - S'^T k);  S = S' + k u^T;  o = scale S^T q
// Column j of the update needs only column j of S plus the scalars q.k and beta, so a thread
// owns four adjacent columns (one float4, coalesced along a row) of a slice of rows; the two
// column sums S'^T k and S'^T q are reduced across the row slices in shared memory. The state
// is read once and written once: 128 KiB of HBM traffic per head against ~0.5 KiB of inputs,
// so the kernel is HBM-bound and only needs enough bytes in flight per SM.
#include "lad_common.cuh"

namespace {

using lad::dev::bf16_to_f32;
using lad::dev::f32_to_bf16;

constexpr int kD = 128;                     // d_k = d_v
constexpr int kThreads = 256;               // 8 warps
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerWarp = kD / kWarps;   // 16 rows of 128 columns per warp
constexpr int kVec = kD / 4;                // float4 per row (one per lane)

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ void fma4(float4 &acc, float a, const float4 &x) {
    acc.x = fmaf(a, x.x, acc.x);
    acc.y = fmaf(a, x.y, acc.y);
    acc.z = fmaf(a, x.z, acc.z);
    acc.w = fmaf(a, x.w, acc.w);
}

__device__ __forceinline__ void add4(float4 &acc, const float4 &x) {
    acc.x += x.x;
    acc.y += x.y;
    acc.z += x.z;
    acc.w += x.w;
}

// The short convolution of one head's q, k and v channels, fused in front of the step (see
// kda_conv_decode_step): raw token x [B][3 H 128], tails [B][3][3 H 128], taps [3 H 128][4].
struct ConvIn {
    const uint16_t *x;
    uint16_t *tail;
    const uint16_t *w;
    const uint16_t *bias;
    int silu;
};

template <bool kOutF32, bool kFusedConv>
__global__ void __launch_bounds__(kThreads, 2)
kda_decode_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k, const uint16_t *__restrict__ v,
                  long long qkv_stride, const float *__restrict__ alpha, const float *__restrict__ beta,
                  float *__restrict__ S, void *__restrict__ o, int H, float scale, int l2norm, ConvIn cv) {
    const int bh = blockIdx.x;
    const int b = bh / H;
    const int h = bh - b * H;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;

    // Issue the 16 state loads first so their latency overlaps everything below.
    float4 *mine = reinterpret_cast<float4 *>(S + static_cast<size_t>(bh) * kD * kD) +
                   static_cast<size_t>(warp * kRowsPerWarp) * kVec + lane;
    float4 s[kRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) s[r] = __ldcs(mine + r * kVec);

    __shared__ float sq[kD], sk[kD], sv[kD], sa[kD];
    __shared__ float4 red_k[kWarps][kVec], red_q[kWarps][kVec];

    if constexpr (kFusedConv) {
        // y = taps . (tail, x) (+ bias), SiLU; kept in fp32; the tail shifts in place. Threads
        // 0-127 take this head's q and k channels, threads 128-255 its v channels.
        const size_t cch = static_cast<size_t>(3) * H * kD;
        const uint16_t *xb = cv.x + static_cast<size_t>(b) * cch;
        uint16_t *tb = cv.tail + static_cast<size_t>(b) * 3 * cch;
        auto conv = [&](size_t c) -> float {
            const uint16_t xr = xb[c], t0 = tb[c], t1 = tb[cch + c], t2 = tb[2 * cch + c];
            const uint2 wv = *reinterpret_cast<const uint2 *>(cv.w + c * 4);
            const float2 w01 = lad::dev::bf16x2_to_f32(wv.x), w23 = lad::dev::bf16x2_to_f32(wv.y);
            float acc = w01.x * bf16_to_f32(t0);
            acc = fmaf(w01.y, bf16_to_f32(t1), acc);
            acc = fmaf(w23.x, bf16_to_f32(t2), acc);
            acc = fmaf(w23.y, bf16_to_f32(xr), acc);
            if (cv.bias) acc += bf16_to_f32(cv.bias[c]);
            if (cv.silu) acc = acc / (1.f + expf(-acc));
            tb[c] = t1;
            tb[cch + c] = t2;
            tb[2 * cch + c] = xr;
            return acc;
        };
        const size_t hc = static_cast<size_t>(h) * kD;
        if (threadIdx.x < kD) {
            const int i = threadIdx.x;
            sq[i] = conv(hc + i);
            sk[i] = conv(static_cast<size_t>(H) * kD + hc + i);
            sa[i] = alpha[static_cast<size_t>(bh) * kD + i];
        } else {
            const int i = threadIdx.x - kD;
            sv[i] = conv(static_cast<size_t>(2) * H * kD + hc + i);
        }
    } else {
        const size_t row = static_cast<size_t>(b) * qkv_stride + static_cast<size_t>(h) * kD;
        if (threadIdx.x < kD) {
            const int i = threadIdx.x;
            sq[i] = bf16_to_f32(q[row + i]);
            sk[i] = bf16_to_f32(k[row + i]);
            sv[i] = bf16_to_f32(v[row + i]);
            sa[i] = alpha[static_cast<size_t>(bh) * kD + i];
        }
    }
    const float bt = beta[bh];
    __syncthreads();

    // q.k, and the inverse norms when normalising; each warp reduces them itself.
    float qq = 0.f, kk = 0.f, qk = 0.f;
#pragma unroll
    for (int i = lane; i < kD; i += 32) {
        const float a = sq[i], c = sk[i];
        qq = fmaf(a, a, qq);
        kk = fmaf(c, c, kk);
        qk = fmaf(a, c, qk);
    }
    qq = warp_sum(qq);
    kk = warp_sum(kk);
    qk = warp_sum(qk);
    float rq = 1.f, rk = 1.f;
    if (l2norm) {
        rq = rsqrtf(qq + 1e-6f);
        rk = rsqrtf(kk + 1e-6f);
    }
    qk *= rq * rk;

    // S' = Diag(alpha) S and this warp's share of S'^T k and S'^T q.
    float4 wk = make_float4(0.f, 0.f, 0.f, 0.f), wq = wk;
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        const int i = warp * kRowsPerWarp + r;
        const float a = sa[i];
        s[r].x *= a;
        s[r].y *= a;
        s[r].z *= a;
        s[r].w *= a;
        fma4(wk, sk[i] * rk, s[r]);
        fma4(wq, sq[i] * rq, s[r]);
    }
    red_k[warp][lane] = wk;
    red_q[warp][lane] = wq;
    __syncthreads();
    float4 W = red_k[0][lane], Q = red_q[0][lane];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
        add4(W, red_k[w][lane]);
        add4(Q, red_q[w][lane]);
    }

    // u = beta (v - S'^T k), then the write S = S' + k u^T.
    const float4 vv = reinterpret_cast<const float4 *>(sv)[lane];
    float4 u;
    u.x = bt * (vv.x - W.x);
    u.y = bt * (vv.y - W.y);
    u.z = bt * (vv.z - W.z);
    u.w = bt * (vv.w - W.w);
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        const int i = warp * kRowsPerWarp + r;
        fma4(s[r], sk[i] * rk, u);
        __stcs(mine + r * kVec, s[r]);
    }

    // o = scale S^T q = scale (S'^T q + (k.q) u)
    if (warp == 0) {
        float4 ov;
        ov.x = scale * fmaf(qk, u.x, Q.x);
        ov.y = scale * fmaf(qk, u.y, Q.y);
        ov.z = scale * fmaf(qk, u.z, Q.z);
        ov.w = scale * fmaf(qk, u.w, Q.w);
        if constexpr (kOutF32) {
            reinterpret_cast<float4 *>(static_cast<float *>(o) + static_cast<size_t>(bh) * kD)[lane] = ov;
        } else {
            uint2 pk;
            pk.x = static_cast<uint32_t>(f32_to_bf16(ov.x)) | (static_cast<uint32_t>(f32_to_bf16(ov.y)) << 16);
            pk.y = static_cast<uint32_t>(f32_to_bf16(ov.z)) | (static_cast<uint32_t>(f32_to_bf16(ov.w)) << 16);
            reinterpret_cast<uint2 *>(static_cast<uint16_t *>(o) + static_cast<size_t>(bh) * kD)[lane] = pk;
        }
    }
}

// T tokens of the same recurrence per state pass (speculative verification: one token plus the
// drafts). The state stays in the registers of K2's layout between tokens; each token costs one
// shared-memory reduction of S'^T k and S'^T q (double-buffered, so one barrier per token).
constexpr int kMaxMultiTokens = 8;

template <bool kOutF32>
__global__ void __launch_bounds__(kThreads, 2)
kda_decode_multi_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                        const uint16_t *__restrict__ v, const float *__restrict__ alpha,
                        const float *__restrict__ beta, float *__restrict__ S, void *__restrict__ o,
                        const int *__restrict__ n_tokens, int B, int T, int H, float scale, int l2norm,
                        int write_state) {
    const int bh = blockIdx.x;
    const int b = bh / H;
    const int h = bh - b * H;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;

    float4 *mine = reinterpret_cast<float4 *>(S + static_cast<size_t>(bh) * kD * kD) +
                   static_cast<size_t>(warp * kRowsPerWarp) * kVec + lane;
    float4 s[kRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) s[r] = __ldcs(mine + r * kVec);

    __shared__ float sq[kMaxMultiTokens][kD], sk[kMaxMultiTokens][kD], sv[kMaxMultiTokens][kD],
        sa[kMaxMultiTokens][kD];
    __shared__ float sb[kMaxMultiTokens], s_rq[kMaxMultiTokens], s_rk[kMaxMultiTokens], s_qk[kMaxMultiTokens];
    __shared__ float4 red_k[2][kWarps][kVec], red_q[2][kWarps][kVec];

    int n = T;
    if (n_tokens) n = min(max(n_tokens[b], 0), T);

    // token t of (b, h): inputs at ((b*T + t)*H + h) rows of 128
    for (int i = threadIdx.x; i < n * kD; i += kThreads) {
        const int t = i / kD, c = i - t * kD;
        const size_t row = (static_cast<size_t>(b) * T + t) * H + h;
        sq[t][c] = bf16_to_f32(q[row * kD + c]);
        sk[t][c] = bf16_to_f32(k[row * kD + c]);
        sv[t][c] = bf16_to_f32(v[row * kD + c]);
        sa[t][c] = alpha[row * kD + c];
    }
    if (threadIdx.x < n) sb[threadIdx.x] = beta[(static_cast<size_t>(b) * T + threadIdx.x) * H + h];
    __syncthreads();
    // warp t: the norms and q.k of token t
    if (warp < n) {
        float qq = 0.f, kk = 0.f, qk = 0.f;
#pragma unroll
        for (int i = lane; i < kD; i += 32) {
            const float a = sq[warp][i], c = sk[warp][i];
            qq = fmaf(a, a, qq);
            kk = fmaf(c, c, kk);
            qk = fmaf(a, c, qk);
        }
        qq = warp_sum(qq);
        kk = warp_sum(kk);
        qk = warp_sum(qk);
        float rq = 1.f, rk = 1.f;
        if (l2norm) {
            rq = rsqrtf(qq + 1e-6f);
            rk = rsqrtf(kk + 1e-6f);
        }
        if (lane == 0) {
            s_rq[warp] = rq;
            s_rk[warp] = rk;
            s_qk[warp] = qk * rq * rk;
        }
    }
    __syncthreads();

    for (int t = 0; t < n; ++t) {
        const float rq = s_rq[t], rk = s_rk[t];
        float4 wk = make_float4(0.f, 0.f, 0.f, 0.f), wq = wk;
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const int i = warp * kRowsPerWarp + r;
            const float a = sa[t][i];
            s[r].x *= a;
            s[r].y *= a;
            s[r].z *= a;
            s[r].w *= a;
            fma4(wk, sk[t][i] * rk, s[r]);
            fma4(wq, sq[t][i] * rq, s[r]);
        }
        // buffer t&1 was last read before the previous token's barrier, which every warp has passed
        red_k[t & 1][warp][lane] = wk;
        red_q[t & 1][warp][lane] = wq;
        __syncthreads();
        float4 W = red_k[t & 1][0][lane], Q = red_q[t & 1][0][lane];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) {
            add4(W, red_k[t & 1][w][lane]);
            add4(Q, red_q[t & 1][w][lane]);
        }
        const float bt = sb[t];
        const float4 vv = reinterpret_cast<const float4 *>(sv[t])[lane];
        float4 u;
        u.x = bt * (vv.x - W.x);
        u.y = bt * (vv.y - W.y);
        u.z = bt * (vv.z - W.z);
        u.w = bt * (vv.w - W.w);
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) fma4(s[r], sk[t][warp * kRowsPerWarp + r] * rk, u);
        if (o && warp == (t & (kWarps - 1))) {
            const float qk = s_qk[t];
            float4 ov;
            ov.x = scale * fmaf(qk, u.x, Q.x);
            ov.y = scale * fmaf(qk, u.y, Q.y);
            ov.z = scale * fmaf(qk, u.z, Q.z);
            ov.w = scale * fmaf(qk, u.w, Q.w);
            const size_t orow = (static_cast<size_t>(b) * T + t) * H + h;
            if constexpr (kOutF32) {
                reinterpret_cast<float4 *>(static_cast<float *>(o) + orow * kD)[lane] = ov;
            } else {
                uint2 pk;
                pk.x = static_cast<uint32_t>(f32_to_bf16(ov.x)) | (static_cast<uint32_t>(f32_to_bf16(ov.y)) << 16);
                pk.y = static_cast<uint32_t>(f32_to_bf16(ov.z)) | (static_cast<uint32_t>(f32_to_bf16(ov.w)) << 16);
                reinterpret_cast<uint2 *>(static_cast<uint16_t *>(o) + orow * kD)[lane] = pk;
            }
        }
    }
    if (write_state && n > 0) {
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) __stcs(mine + r * kVec, s[r]);
    }
}

}  // namespace

extern "C" int kda_decode_step(const lad_bf16 *q, const lad_bf16 *k, const lad_bf16 *v, long long qkv_batch_stride,
                               const float *alpha, const float *beta, float *S, void *o, int B, int H, int dk,
                               int dv, float scale, unsigned flags, void *stream) {
    using lad::set_error;
    if (B < 0 || H < 0) return set_error(LAD_EINVAL, "kda_decode_step: negative B or H");
    if (dk != kD || dv != kD) return set_error(LAD_EUNSUPPORTED, "kda_decode_step: dk = dv = 128 only");
    if (B == 0 || H == 0) return LAD_OK;
    if (!q || !k || !v || !alpha || !beta || !S || !o)
        return set_error(LAD_EINVAL, "kda_decode_step: null pointer");
    if (qkv_batch_stride < 0) return set_error(LAD_EINVAL, "kda_decode_step: negative qkv_batch_stride");
    const long long stride = qkv_batch_stride ? qkv_batch_stride : static_cast<long long>(H) * kD;
    if (stride < static_cast<long long>(H) * kD)
        return set_error(LAD_EINVAL, "kda_decode_step: qkv_batch_stride %lld < H*128", stride);
    if (!lad::aligned(S, 16)) return set_error(LAD_EUNSUPPORTED, "kda_decode_step: S must be 16-byte aligned");
    const bool f32 = (flags & LAD_FLAG_OUT_FP32) != 0;
    if (!lad::aligned(o, f32 ? 16 : 8)) return set_error(LAD_EUNSUPPORTED, "kda_decode_step: o misaligned");
    if (flags & ~(LAD_FLAG_OUT_FP32 | LAD_FLAG_L2NORM_QK))
        return set_error(LAD_EINVAL, "kda_decode_step: unknown flags 0x%x", flags);
    const long long blocks = static_cast<long long>(B) * H;
    if (blocks > 0x7fffffffLL) return set_error(LAD_EUNSUPPORTED, "kda_decode_step: B*H too large");
    const int l2 = (flags & LAD_FLAG_L2NORM_QK) ? 1 : 0;
    cudaStream_t s = lad::as_stream(stream);
    const ConvIn none{nullptr, nullptr, nullptr, nullptr, 0};
    if (f32)
        kda_decode_kernel<true, false><<<static_cast<unsigned>(blocks), kThreads, 0, s>>>(q, k, v, stride, alpha, beta,
                                                                                          S, o, H, scale, l2, none);
    else
        kda_decode_kernel<false, false><<<static_cast<unsigned>(blocks), kThreads, 0, s>>>(q, k, v, stride, alpha, beta,
                                                                                           S, o, H, scale, l2, none);
    return lad::check_launch("kda_decode_step");
}

extern "C" int kda_conv_decode_step(const lad_bf16 *x, lad_bf16 *conv_tail, const lad_bf16 *conv_w,
                                    const lad_bf16 *conv_bias, const float *alpha, const float *beta, float *S, void *o,
                                    int B, int H, int dk, int dv, int K, float scale, unsigned flags, void *stream) {
    using lad::set_error;
    if (B < 0 || H < 0) return set_error(LAD_EINVAL, "kda_conv_decode_step: negative B or H");
    if (dk != kD || dv != kD) return set_error(LAD_EUNSUPPORTED, "kda_conv_decode_step: dk = dv = 128 only");
    if (K != 4) return set_error(LAD_EUNSUPPORTED, "kda_conv_decode_step: K = 4 only");
    if (flags & ~(LAD_FLAG_OUT_FP32 | LAD_FLAG_L2NORM_QK | LAD_FLAG_SILU))
        return set_error(LAD_EINVAL, "kda_conv_decode_step: unknown flags 0x%x", flags);
    if (B == 0 || H == 0) return LAD_OK;
    if (!x || !conv_tail || !conv_w || !alpha || !beta || !S || !o)
        return set_error(LAD_EINVAL, "kda_conv_decode_step: null pointer");
    if (!lad::aligned(S, 16) || !lad::aligned(conv_w, 8))
        return set_error(LAD_EUNSUPPORTED, "kda_conv_decode_step: S 16-byte and conv_w 8-byte aligned");
    const bool f32 = (flags & LAD_FLAG_OUT_FP32) != 0;
    if (!lad::aligned(o, f32 ? 16 : 8)) return set_error(LAD_EUNSUPPORTED, "kda_conv_decode_step: o misaligned");
    const long long blocks = static_cast<long long>(B) * H;
    if (blocks > 0x7fffffffLL) return set_error(LAD_EUNSUPPORTED, "kda_conv_decode_step: B*H too large");
    const int l2 = (flags & LAD_FLAG_L2NORM_QK) ? 1 : 0;
    const ConvIn cv{x, conv_tail, conv_w, conv_bias, (flags & LAD_FLAG_SILU) ? 1 : 0};
    cudaStream_t s = lad::as_stream(stream);
    if (f32)
        kda_decode_kernel<true, true><<<static_cast<unsigned>(blocks), kThreads, 0, s>>>(
            nullptr, nullptr, nullptr, 0, alpha, beta, S, o, H, scale, l2, cv);
    else
        kda_decode_kernel<false, true><<<static_cast<unsigned>(blocks), kThreads, 0, s>>>(
            nullptr, nullptr, nullptr, 0, alpha, beta, S, o, H, scale, l2, cv);
    return lad::check_launch("kda_conv_decode_step");
}

extern "C" int kda_decode_multi(const lad_bf16 *q, const lad_bf16 *k, const lad_bf16 *v, const float *alpha,
                                const float *beta, float *S, void *o, const int *n_tokens, int B, int T, int H, int dk,
                                int dv, float scale, unsigned flags, void *stream) {
    using lad::set_error;
    if (B < 0 || H < 0 || T < 0) return set_error(LAD_EINVAL, "kda_decode_multi: negative B, T or H");
    if (dk != kD || dv != kD) return set_error(LAD_EUNSUPPORTED, "kda_decode_multi: dk = dv = 128 only");
    if (T > kMaxMultiTokens)
        return set_error(LAD_EUNSUPPORTED, "kda_decode_multi: at most %d tokens per call", kMaxMultiTokens);
    if (flags & ~(LAD_FLAG_OUT_FP32 | LAD_FLAG_L2NORM_QK | LAD_FLAG_KEEP_STATE))
        return set_error(LAD_EINVAL, "kda_decode_multi: unknown flags 0x%x", flags);
    if (B == 0 || H == 0 || T == 0) return LAD_OK;
    if (!q || !k || !v || !alpha || !beta || !S) return set_error(LAD_EINVAL, "kda_decode_multi: null pointer");
    if (!lad::aligned(S, 16)) return set_error(LAD_EUNSUPPORTED, "kda_decode_multi: S must be 16-byte aligned");
    const bool f32 = (flags & LAD_FLAG_OUT_FP32) != 0;
    if (o && !lad::aligned(o, f32 ? 16 : 8)) return set_error(LAD_EUNSUPPORTED, "kda_decode_multi: o misaligned");
    const long long blocks = static_cast<long long>(B) * H;
    if (blocks > 0x7fffffffLL) return set_error(LAD_EUNSUPPORTED, "kda_decode_multi: B*H too large");
    const int l2 = (flags & LAD_FLAG_L2NORM_QK) ? 1 : 0;
    const int write_state = (flags & LAD_FLAG_KEEP_STATE) ? 0 : 1;
    cudaStream_t s = lad::as_stream(stream);
    if (f32)
        kda_decode_multi_kernel<true><<<static_cast<unsigned>(blocks), kThreads, 0, s>>>(
            q, k, v, alpha, beta, S, o, n_tokens, B, T, H, scale, l2, write_state);
    else
        kda_decode_multi_kernel<false><<<static_cast<unsigned>(blocks), kThreads, 0, s>>>(
            q, k, v, alpha, beta, S, o, n_tokens, B, T, H, scale, l2, write_state);
    return lad::check_launch("kda_decode_multi");
}
