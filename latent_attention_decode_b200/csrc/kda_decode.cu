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
#include <algorithm>
#include <mutex>

#include "sm100_ptx.cuh"

namespace {

__device__ int g_kda_error = 0;

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

// fma4 as two packed fp32 pair instructions (each lane rounded as the scalar FMA): the same bits
__device__ __forceinline__ void fma4p(float4 &acc, float a, const float4 &x) {
    const float2 lo = lad::ptx::fma2(make_float2(a, a), make_float2(x.x, x.y), make_float2(acc.x, acc.y));
    const float2 hi = lad::ptx::fma2(make_float2(a, a), make_float2(x.z, x.w), make_float2(acc.z, acc.w));
    acc = make_float4(lo.x, lo.y, hi.x, hi.y);
}

__device__ __forceinline__ void add4(float4 &acc, const float4 &x) {
    acc.x += x.x;
    acc.y += x.y;
    acc.z += x.z;
    acc.w += x.w;
}

// Output gate of the head (kda_conv_decode_step_gated), applied to o in the epilogue:
// o <- o / sqrt(mean(o^2) + eps) * w * sigmoid(g), g [B][H][128] bf16, w [128] fp32 or null.
struct GateIn {
    const uint16_t *g;
    const float *w;
    float eps;
};

// The short convolution of one head's q, k and v channels, fused in front of the step (see
// kda_conv_decode_step): raw token x [B][3 H 128], tails [B][3][3 H 128], taps [3 H 128][4].
struct ConvIn {
    const uint16_t *x;
    uint16_t *tail;
    const uint16_t *w;
    const uint16_t *bias;
    int silu;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// kPair (small batches): a CTA updates two heads, bh = blockIdx.x and bh + gridDim.x. With one
// head per CTA and B * H between one and two times the resident CTAs (8 x 64 heads on 296 slots),
// the CTAs of the second wave start only as the first wave's finish, and the waves load, reduce
// and store in step, so HBM idles between the phases. Here the second head's 64 KiB state comes
// into shared memory by one bulk copy (the copy engine, not the load/store units, which the
// first head's 16 loads per thread keep busy) while the first head is loaded into registers, so
// every state byte of the launch is requested at once; the second head then runs from shared
// memory while the first head's stores drain. The copy's wait is bounded: if it runs out, the
// second head is left untouched and device error 0x501 is recorded.
// dynamic shared memory of the paired kernel: the second head's 64 KiB state, then its copy's
// mbarrier and abort flag, the whole region aligned to 128 bytes by hand (the dynamic region
// starts wherever the static shared variables end, which need not be 16-byte aligned)
constexpr int kPairStateBytes = kD * kD * 4;
constexpr int kPairSmemBytes = kPairStateBytes + 16 + 128;

template <bool kOutF32, bool kFusedConv, bool kPair>
__global__ void __launch_bounds__(kThreads, 2)
kda_decode_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k, const uint16_t *__restrict__ v,
                  long long qkv_stride, const float *__restrict__ alpha, const float *__restrict__ beta,
                  float *__restrict__ S, void *__restrict__ o, int H, float scale, int l2norm, ConvIn cv,
                  GateIn gi, int units) {
    constexpr int kUnits = kPair ? 2 : 1;
    extern __shared__ uint8_t pair_raw[];  // kPair: the second head's state (aligned below)
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int bh0 = blockIdx.x;
    const int bh1 = kPair ? bh0 + static_cast<int>(gridDim.x) : units;
    const bool has1 = kPair && bh1 < units;  // uniform over the CTA

    auto state_of = [&](int bh) {
        return reinterpret_cast<float4 *>(S + static_cast<size_t>(bh) * kD * kD) +
               static_cast<size_t>(warp * kRowsPerWarp) * kVec + lane;
    };
    // Issue the 16 state loads first so their latency overlaps everything below.
    float4 s[kRowsPerWarp];
    {
        const float4 *mine = state_of(bh0);
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) s[r] = __ldcs(mine + r * kVec);
    }
    uint8_t *pair_slots =
        reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(pair_raw) + 127) & ~static_cast<uintptr_t>(127));
    const uint32_t bar = static_cast<uint32_t>(__cvta_generic_to_shared(pair_slots + kPairStateBytes));
    volatile int *pair_abort = reinterpret_cast<volatile int *>(pair_slots + kPairStateBytes + 8);
    if (has1 && threadIdx.x == 0) {
        *pair_abort = 0;
        lad::ptx::mbar_init(bar, 1);
        lad::ptx::mbar_fence_init();
        lad::ptx::mbar_arrive_tx_raw(bar, kD * kD * 4);
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                static_cast<uint32_t>(__cvta_generic_to_shared(pair_slots))),
            "l"(reinterpret_cast<uint64_t>(S + static_cast<size_t>(bh1) * kD * kD)), "r"(kD * kD * 4), "r"(bar)
            : "memory");
    }
    // Launched as a programmatic dependent (LAD_FLAG_OVERLAP_PREV), the CTAs start while the kernel
    // before this one on the stream still runs: only the state reads above are issued before this
    // wait, and everything else (the token inputs, the conv tails, every write) comes after it.
    // Then the next such launch may start; its CTAs take SMs as these ones leave. Launched
    // normally, the wait returns at once and the trigger does nothing.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    __shared__ float sq[kUnits][kD], sk[kUnits][kD], sv[kUnits][kD], sa[kUnits][kD];
    __shared__ float4 red_k[kWarps][kVec], red_q[kWarps][kVec];

    // the heads' q, k, v (through the fused conv, or as given) and alpha into their slots. With the
    // fused conv, every input of every conv this thread does (q and k channels for threads 0-127, v
    // channels for 128-255, of each of the CTA's heads) is loaded first, and only then are the
    // outputs computed and the tails shifted: a tail store must not come between two convs' loads,
    // or each conv would wait a full memory round trip behind the state stream
    auto inputs = [&]() {
        const int nheads = has1 ? 2 : 1;
        if constexpr (kFusedConv) {
            const size_t cch = static_cast<size_t>(3) * H * kD;
            const bool qk = threadIdx.x < kD;
            const int i = qk ? threadIdx.x : threadIdx.x - kD;
            uint16_t xr[kUnits][2], t0[kUnits][2], t1[kUnits][2], t2[kUnits][2], bs[kUnits][2];
            uint2 wv[kUnits][2];
            float al[kUnits];
            size_t chan[kUnits][2];
#pragma unroll
            for (int u = 0; u < kUnits; ++u) {
                if (u < nheads) {
                    const int bh = u == 0 ? bh0 : bh1;
                    const int b = bh / H, h = bh - b * H;
                    const size_t hc = static_cast<size_t>(h) * kD;
                    const uint16_t *xb = cv.x + static_cast<size_t>(b) * cch;
                    const uint16_t *tb = cv.tail + static_cast<size_t>(b) * 3 * cch;
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        if (j == 0 || qk) {
                            const size_t c = qk ? static_cast<size_t>(j) * H * kD + hc + i
                                                : static_cast<size_t>(2) * H * kD + hc + i;
                            chan[u][j] = static_cast<size_t>(b) * cch + c;
                            xr[u][j] = xb[c];
                            t0[u][j] = tb[c];
                            t1[u][j] = tb[cch + c];
                            t2[u][j] = tb[2 * cch + c];
                            wv[u][j] = *reinterpret_cast<const uint2 *>(cv.w + c * 4);
                            bs[u][j] = cv.bias ? cv.bias[c] : static_cast<uint16_t>(0);
                        }
                    }
                    al[u] = qk ? alpha[static_cast<size_t>(bh) * kD + i] : 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < kUnits; ++u) {
                if (u < nheads) {
                    const int b = (u == 0 ? bh0 : bh1) / H;
                    uint16_t *tb = cv.tail + static_cast<size_t>(b) * 3 * cch;
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        if (j == 0 || qk) {
                            // y = taps . (tail, x) (+ bias), SiLU; kept in fp32; the tail shifts in place
                            const float2 w01 = lad::dev::bf16x2_to_f32(wv[u][j].x),
                                         w23 = lad::dev::bf16x2_to_f32(wv[u][j].y);
                            float acc = w01.x * bf16_to_f32(t0[u][j]);
                            acc = fmaf(w01.y, bf16_to_f32(t1[u][j]), acc);
                            acc = fmaf(w23.x, bf16_to_f32(t2[u][j]), acc);
                            acc = fmaf(w23.y, bf16_to_f32(xr[u][j]), acc);
                            if (cv.bias) acc += bf16_to_f32(bs[u][j]);
                            if (cv.silu) acc = acc / (1.f + expf(-acc));
                            const size_t c = chan[u][j] - static_cast<size_t>(b) * cch;
                            tb[c] = t1[u][j];
                            tb[cch + c] = t2[u][j];
                            tb[2 * cch + c] = xr[u][j];
                            if (!qk)
                                sv[u][i] = acc;
                            else if (j == 0)
                                sq[u][i] = acc;
                            else
                                sk[u][i] = acc;
                        }
                    }
                    if (qk) sa[u][i] = al[u];
                }
            }
        } else {
#pragma unroll
            for (int u = 0; u < kUnits; ++u) {
                if (u < nheads && threadIdx.x < kD) {
                    const int bh = u == 0 ? bh0 : bh1;
                    const int b = bh / H, h = bh - b * H;
                    const size_t row = static_cast<size_t>(b) * qkv_stride + static_cast<size_t>(h) * kD;
                    const int i = threadIdx.x;
                    sq[u][i] = bf16_to_f32(q[row + i]);
                    sk[u][i] = bf16_to_f32(k[row + i]);
                    sv[u][i] = bf16_to_f32(v[row + i]);
                    sa[u][i] = alpha[static_cast<size_t>(bh) * kD + i];
                }
            }
        }
    };

    // one head's update from the state in s (slot u of the inputs); ends with the new state
    // stored and o written
    auto update = [&](int u, int bh) {
        const float bt = beta[bh];
        // the output gate's logits and norm weight (4 of each per lane of warp 0, which computes the
        // outputs): into registers now, used only in the epilogue, so nothing waits for them
        uint2 gate4 = make_uint2(0u, 0u);
        float4 w4 = make_float4(1.f, 1.f, 1.f, 1.f);
        if (gi.g && warp == 0) {
            gate4 = reinterpret_cast<const uint2 *>(gi.g + static_cast<size_t>(bh) * kD)[lane];
            if (gi.w) w4 = reinterpret_cast<const float4 *>(gi.w)[lane];
        }
        // q.k, and the inverse norms when normalising; each warp reduces them itself.
        float qq = 0.f, kk = 0.f, qk = 0.f;
#pragma unroll
        for (int i = lane; i < kD; i += 32) {
            const float a = sq[u][i], c = sk[u][i];
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
            const float a = sa[u][i];
            s[r].x *= a;
            s[r].y *= a;
            s[r].z *= a;
            s[r].w *= a;
            fma4(wk, sk[u][i] * rk, s[r]);
            fma4(wq, sq[u][i] * rq, s[r]);
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
        const float4 vv = reinterpret_cast<const float4 *>(sv[u])[lane];
        float4 uu;
        uu.x = bt * (vv.x - W.x);
        uu.y = bt * (vv.y - W.y);
        uu.z = bt * (vv.z - W.z);
        uu.w = bt * (vv.w - W.w);
        float4 *mine = state_of(bh);
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const int i = warp * kRowsPerWarp + r;
            fma4(s[r], sk[u][i] * rk, uu);
            __stcs(mine + r * kVec, s[r]);
        }

        // o = scale S^T q = scale (S'^T q + (k.q) u)
        if (warp == 0) {
            float4 ov;
            ov.x = scale * fmaf(qk, uu.x, Q.x);
            ov.y = scale * fmaf(qk, uu.y, Q.y);
            ov.z = scale * fmaf(qk, uu.z, Q.z);
            ov.w = scale * fmaf(qk, uu.w, Q.w);
            if (gi.g) {
                // gated RMSNorm over the head's 128 outputs (4 per lane)
                const float ss = warp_sum(ov.x * ov.x + ov.y * ov.y + ov.z * ov.z + ov.w * ov.w);
                const float inv = rsqrtf(ss * (1.f / kD) + gi.eps);
                const float2 g01 = lad::dev::bf16x2_to_f32(gate4.x), g23 = lad::dev::bf16x2_to_f32(gate4.y);
                ov.x *= inv * w4.x / (1.f + __expf(-g01.x));
                ov.y *= inv * w4.y / (1.f + __expf(-g01.y));
                ov.z *= inv * w4.z / (1.f + __expf(-g23.x));
                ov.w *= inv * w4.w / (1.f + __expf(-g23.y));
            }
            if constexpr (kOutF32) {
                reinterpret_cast<float4 *>(static_cast<float *>(o) + static_cast<size_t>(bh) * kD)[lane] = ov;
            } else {
                uint2 pk;
                pk.x = static_cast<uint32_t>(f32_to_bf16(ov.x)) | (static_cast<uint32_t>(f32_to_bf16(ov.y)) << 16);
                pk.y = static_cast<uint32_t>(f32_to_bf16(ov.z)) | (static_cast<uint32_t>(f32_to_bf16(ov.w)) << 16);
                reinterpret_cast<uint2 *>(static_cast<uint16_t *>(o) + static_cast<size_t>(bh) * kD)[lane] = pk;
            }
        }
    };

    inputs();
    __syncthreads();
    update(0, bh0);
    if constexpr (kPair) {
        if (has1) {
            // the second head from shared memory (the state's own layout: this thread's rows and
            // float4 of columns), then a barrier before the reduction buffers and gate inputs are reused
            const bool landed = lad::ptx::wait_bar(bar, 0, pair_abort, &g_kda_error, lad::kErrKdaPair);
            const float4 *rows = reinterpret_cast<const float4 *>(pair_slots) +
                                 static_cast<size_t>(warp * kRowsPerWarp) * kVec + lane;
#pragma unroll
            for (int r = 0; r < kRowsPerWarp; ++r) s[r] = rows[r * kVec];
            if (__syncthreads_and(landed)) {
                update(1, bh1);
            } else if (threadIdx.x == 0) {
                // the copy may still be in flight: give it one more bounded wait before the CTA
                // (and its shared memory) goes away
                const uint64_t t0 = lad::dev::globaltimer_ns();
                while (!lad::ptx::mbar_try_wait(bar, 0) && lad::dev::globaltimer_ns() - t0 < lad::dev::kWaitLimitNs) {
                }
            }
        }
    }
}

// T tokens of the same recurrence per state pass (speculative verification: one token plus the
// drafts). Each token adds a dependent chain (decay, column sums S'^T k and S'^T q across the
// row slices, update) of a few microseconds per head; launched one head per CTA, the CTAs of an
// SM would load, compute and store in step and leave HBM idle during the chains. So the kernel is
// persistent (two CTAs per SM walk the heads with a stride of the grid) and prefetches: while
// head i's tokens run in registers, each thread's cp.async copies bring its slice of head i+1's
// state into its own slots of shared memory (read back by the same thread only, so no barrier
// is needed for them), and head i+1's token inputs land by cp.async in the other of two input
// buffers. Thread layout: warp w owns
// columns 16w..16w+15 over all 128 rows; lane = (row group lane/4, float4 of columns lane%4) and
// holds rows 8m + lane/4 (m = 0..15). A warp instruction then reads 8 rows x 64 contiguous bytes,
// and the column sums S'^T k and S'^T q reduce over the 8 row groups with three shuffles: the
// warps never wait for one another inside the token loop.
constexpr int kMaxMultiTokens = 8;
constexpr float kLazyMin = 1e-20f;  // smallest cumulative decay the lazy form takes (1 / L <= 1e20)
constexpr int kMultiCtasPerSm = 2;
constexpr int kPiecesPerToken = 80;  // 16-byte pieces of one token's inputs: q 16, k 16, v 16, alpha 32

// dynamic shared memory: state slots, per-token scalars, raw inputs, per-row factors
constexpr int kMOffState = 0;                                   // [16 rows][256 threads] float4
constexpr int kMOffScal = kMOffState + kRowsPerWarp * kThreads * 16;  // beta, 1/|q|, 1/|k|, q.k per token
constexpr int kMOffBeta = kMOffScal + 4 * kMaxMultiTokens * 4;      // [2 buffers][8] beta
constexpr int kMOffRaw = kMOffBeta + 2 * kMaxMultiTokens * 4;       // [2 buffers] per token: q,k,v bf16, alpha fp32
constexpr int kRawTokenBytes = 3 * kD * 2 + kD * 4;                 // 1,280
__host__ __device__ constexpr int multi_smem_bytes(int T) {
    return kMOffRaw + 2 * T * kRawTokenBytes + T * kD * 16 + T * kD * 4;  // + per-row {alpha, k, q}, k
}


// cp.async of head bh's token inputs (tokens 0..n-1) into one input buffer: piece p of token t
// (16 bytes: q, k, v 8 bf16 each, alpha 4 fp32) and beta_t. The caller commits.
__device__ __forceinline__ void prefetch_inputs(uint32_t raw_dst, uint32_t beta_dst, const uint16_t *q,
                                                const uint16_t *k, const uint16_t *v, const float *alpha,
                                                const float *beta, int bh, int H, int T, int n) {
    const int b = bh / H, h = bh - b * H;
    for (int p = threadIdx.x; p < n * kPiecesPerToken; p += kThreads) {
        const int t = p / kPiecesPerToken, c = p - t * kPiecesPerToken;
        const size_t row = ((static_cast<size_t>(b) * T + t) * H + h) * kD;
        const uint32_t dst = raw_dst + t * kRawTokenBytes + (c < 48 ? (c >> 4) * 256 + (c & 15) * 16 : 768 + (c - 48) * 16);
        if (c < 48) {
            const uint16_t *src = c < 16 ? q : (c < 32 ? k : v);
            cp_async16(dst, src + row + 8 * (c & 15));
        } else {
            cp_async16(dst, alpha + row + 4 * (c - 48));
        }
    }
    if (threadIdx.x < n)
        cp_async4(beta_dst + threadIdx.x * 4, beta + (static_cast<size_t>(b) * T + threadIdx.x) * H + h);
}

template <bool kOutF32>
__global__ void __launch_bounds__(kThreads, kMultiCtasPerSm)
kda_decode_multi_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                        const uint16_t *__restrict__ v, const float *__restrict__ alpha,
                        const float *__restrict__ beta, float *__restrict__ S, void *__restrict__ o,
                        const int *__restrict__ n_tokens, int B, int T, int H, float scale, int l2norm,
                        int write_state) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int heads = B * H;
    const uint32_t st_base = static_cast<uint32_t>(__cvta_generic_to_shared(smem + kMOffState)) + tid * 16;
    const float4 *st = reinterpret_cast<const float4 *>(smem + kMOffState) + tid;
    float *s_rq = reinterpret_cast<float *>(smem + kMOffScal);
    float *s_rk = s_rq + kMaxMultiTokens, *s_qk = s_rk + kMaxMultiTokens;
    const uint32_t raw_base = static_cast<uint32_t>(__cvta_generic_to_shared(smem + kMOffRaw));
    const uint32_t beta_base = static_cast<uint32_t>(__cvta_generic_to_shared(smem + kMOffBeta));
    float4 *rowf = reinterpret_cast<float4 *>(smem + kMOffRaw + 2 * T * kRawTokenBytes);  // [t][row]
    float *rowk = reinterpret_cast<float *>(rowf + T * kD);  // [t][row]: k_i / |k| again, for the update

    auto n_of = [&](int bh) { return n_tokens ? min(max(n_tokens[bh / H], 0), T) : T; };
    const int rsub = lane >> 2;  // row group: rows 8m + rsub
    const int cq = lane & 3;     // float4 of columns 16*warp + 4*cq
    // float4 index of (row 8m + rsub, this thread's columns) is m * 8 * kVec + thread_f4
    const int thread_f4 = rsub * kVec + 4 * warp + cq;
    auto prefetch_state = [&](int bh) {
        const float4 *src = reinterpret_cast<const float4 *>(S + static_cast<size_t>(bh) * kD * kD) + thread_f4;
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) cp_async16(st_base + r * kThreads * 16, src + r * 8 * kVec);
        cp_async_commit();
    };

    int bh = blockIdx.x;
    if (bh >= heads) return;
    int n = n_of(bh);
    prefetch_state(bh);
    prefetch_inputs(raw_base, beta_base, q, k, v, alpha, beta, bh, H, T, n);
    cp_async_commit();

    for (int it = 0; bh < heads; ++it) {
        const int b = bh / H, h = bh - b * H;
        const int buf = it & 1;
        const uint8_t *raw = smem + kMOffRaw + buf * T * kRawTokenBytes;  // token t at t * kRawTokenBytes
        const float *s_beta = reinterpret_cast<const float *>(smem + kMOffBeta) + buf * kMaxMultiTokens;
        // 1. this head's state slots and inputs have landed (inputs are read by every thread)
        cp_async_wait_all();
        __syncthreads();
        // 2. warp t: the norms and q.k of token t
        if (warp < n) {
            const uint16_t *tq = reinterpret_cast<const uint16_t *>(raw + warp * kRawTokenBytes);
            const uint2 xq = reinterpret_cast<const uint2 *>(tq)[lane];
            const uint2 xk = reinterpret_cast<const uint2 *>(tq + kD)[lane];
            const float2 q0 = lad::dev::bf16x2_to_f32(xq.x), q1 = lad::dev::bf16x2_to_f32(xq.y);
            const float2 k0 = lad::dev::bf16x2_to_f32(xk.x), k1 = lad::dev::bf16x2_to_f32(xk.y);
            float qq = q0.x * q0.x + q0.y * q0.y + q1.x * q1.x + q1.y * q1.y;
            float kk = k0.x * k0.x + k0.y * k0.y + k1.x * k1.x + k1.y * k1.y;
            float qk = q0.x * k0.x + q0.y * k0.y + q1.x * k1.x + q1.y * k1.y;
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
        // 3. per-row factors of every token. The decays are applied lazily: with L_t = prod_{s<=t}
        //    alpha_s per row, the registers hold S~ = S / L (row-wise), so that token t's column sums
        //    take the coefficients L_t k and L_t q, its update adds (k / L_t) u^T to S~, and only
        //    the final state is multiplied by L (no per-token decay pass over the state). Row
        //    factors {L k, L q, L} and k / L. A head whose L falls below kLazyMin on some row (1 / L
        //    would leave the safe fp32 range) takes the eager form instead: {alpha, k, q} and k.
        bool lazy_ok = true;
        if (tid < kD) {
            const int i = tid;
            float lam = 1.f, lo = 1.f;
            for (int t = 0; t < n; ++t) {
                const uint16_t *tq = reinterpret_cast<const uint16_t *>(raw + t * kRawTokenBytes);
                const float a = reinterpret_cast<const float *>(raw + t * kRawTokenBytes + 768)[i];
                const float kn = bf16_to_f32(tq[kD + i]) * s_rk[t];
                const float qn = bf16_to_f32(tq[i]) * s_rq[t];
                lam *= a;
                lo = fminf(lo, lam);
                rowf[t * kD + i] = make_float4(lam * kn, lam * qn, lam, 0.f);
                rowk[t * kD + i] = kn / lam;
            }
            lazy_ok = lo >= kLazyMin;
        }
        const bool lazy = __syncthreads_and(lazy_ok) != 0;
        if (!lazy) {
            for (int e = tid; e < n * kD; e += kThreads) {
                const int t = e >> 7, i = e & (kD - 1);
                const uint16_t *tq = reinterpret_cast<const uint16_t *>(raw + t * kRawTokenBytes);
                const float a = reinterpret_cast<const float *>(raw + t * kRawTokenBytes + 768)[i];
                const float kn = bf16_to_f32(tq[kD + i]) * s_rk[t];
                rowf[e] = make_float4(a, kn, bf16_to_f32(tq[i]) * s_rq[t], 0.f);
                rowk[e] = kn;
            }
        }
        // 4. this head's state: this thread's own slots
        float4 s[kRowsPerWarp];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) s[r] = st[r * kThreads];
        __syncthreads();
        // 5. prefetch the next head: state into the same slots, inputs into the other buffer (its
        //    last readers finished before the barrier at the end of the previous iteration)
        const int nbh = bh + gridDim.x;
        int nn = 0;
        if (nbh < heads) {
            nn = n_of(nbh);
            prefetch_state(nbh);
            prefetch_inputs(raw_base + (buf ^ 1) * T * kRawTokenBytes, beta_base + (buf ^ 1) * kMaxMultiTokens * 4, q,
                            k, v, alpha, beta, nbh, H, T, nn);
            cp_async_commit();
        }
        // 6. the tokens (lazy decays, or the eager form)
        if (lazy) {
            for (int t = 0; t < n; ++t) {
                const float4 *rf = rowf + t * kD + rsub;
                float4 wk = make_float4(0.f, 0.f, 0.f, 0.f), wq = wk;
                // two halves with a compiler fence between them, so that at most eight row-factor
                // loads are hoisted at a time (all sixteen would not fit next to the state)
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int mm = 0; mm < kRowsPerWarp / 2; ++mm) {
                        const int m = half * (kRowsPerWarp / 2) + mm;
                        const float4 f = rf[8 * m];
                        fma4p(wk, f.x, s[m]);
                        fma4p(wq, f.y, s[m]);
                    }
                    asm volatile("" ::: "memory");
                }
#pragma unroll
                for (int x = 4; x < 32; x <<= 1) {
                    wk.x += __shfl_xor_sync(0xffffffffu, wk.x, x);
                    wk.y += __shfl_xor_sync(0xffffffffu, wk.y, x);
                    wk.z += __shfl_xor_sync(0xffffffffu, wk.z, x);
                    wk.w += __shfl_xor_sync(0xffffffffu, wk.w, x);
                    wq.x += __shfl_xor_sync(0xffffffffu, wq.x, x);
                    wq.y += __shfl_xor_sync(0xffffffffu, wq.y, x);
                    wq.z += __shfl_xor_sync(0xffffffffu, wq.z, x);
                    wq.w += __shfl_xor_sync(0xffffffffu, wq.w, x);
                }
                const float bt = s_beta[t];
                const uint2 xv = reinterpret_cast<const uint2 *>(raw + t * kRawTokenBytes + 512)[4 * warp + cq];
                const float2 v0 = lad::dev::bf16x2_to_f32(xv.x), v1 = lad::dev::bf16x2_to_f32(xv.y);
                float4 u;
                u.x = bt * (v0.x - wk.x);
                u.y = bt * (v0.y - wk.y);
                u.z = bt * (v1.x - wk.z);
                u.w = bt * (v1.y - wk.w);
#pragma unroll
                for (int m = 0; m < kRowsPerWarp; ++m) fma4p(s[m], rowk[t * kD + 8 * m + rsub], u);
                if (o && rsub == 0) {
                    const float qk = s_qk[t];
                    float4 ov;
                    ov.x = scale * fmaf(qk, u.x, wq.x);
                    ov.y = scale * fmaf(qk, u.y, wq.y);
                    ov.z = scale * fmaf(qk, u.z, wq.z);
                    ov.w = scale * fmaf(qk, u.w, wq.w);
                    const size_t orow = ((static_cast<size_t>(b) * T + t) * H + h) * kD;
                    if constexpr (kOutF32) {
                        reinterpret_cast<float4 *>(static_cast<float *>(o) + orow)[4 * warp + cq] = ov;
                    } else {
                        uint2 pk;
                        pk.x = static_cast<uint32_t>(f32_to_bf16(ov.x)) | (static_cast<uint32_t>(f32_to_bf16(ov.y)) << 16);
                        pk.y = static_cast<uint32_t>(f32_to_bf16(ov.z)) | (static_cast<uint32_t>(f32_to_bf16(ov.w)) << 16);
                        reinterpret_cast<uint2 *>(static_cast<uint16_t *>(o) + orow)[4 * warp + cq] = pk;
                    }
                }
            }
        } else {
            for (int t = 0; t < n; ++t) {
                const float4 *rf = rowf + t * kD + rsub;
                float4 wk = make_float4(0.f, 0.f, 0.f, 0.f), wq = wk;
                // two halves with a compiler fence between them, so that at most eight row-factor
                // loads are hoisted at a time (all sixteen would not fit next to the state)
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int mm = 0; mm < kRowsPerWarp / 2; ++mm) {
                        const int m = half * (kRowsPerWarp / 2) + mm;
                        const float4 f = rf[8 * m];
                        s[m].x *= f.x;
                        s[m].y *= f.x;
                        s[m].z *= f.x;
                        s[m].w *= f.x;
                        fma4(wk, f.y, s[m]);
                        fma4(wq, f.z, s[m]);
                    }
                    asm volatile("" ::: "memory");
                }
#pragma unroll
                for (int x = 4; x < 32; x <<= 1) {
                    wk.x += __shfl_xor_sync(0xffffffffu, wk.x, x);
                    wk.y += __shfl_xor_sync(0xffffffffu, wk.y, x);
                    wk.z += __shfl_xor_sync(0xffffffffu, wk.z, x);
                    wk.w += __shfl_xor_sync(0xffffffffu, wk.w, x);
                    wq.x += __shfl_xor_sync(0xffffffffu, wq.x, x);
                    wq.y += __shfl_xor_sync(0xffffffffu, wq.y, x);
                    wq.z += __shfl_xor_sync(0xffffffffu, wq.z, x);
                    wq.w += __shfl_xor_sync(0xffffffffu, wq.w, x);
                }
                const float bt = s_beta[t];
                const uint2 xv = reinterpret_cast<const uint2 *>(raw + t * kRawTokenBytes + 512)[4 * warp + cq];
                const float2 v0 = lad::dev::bf16x2_to_f32(xv.x), v1 = lad::dev::bf16x2_to_f32(xv.y);
                float4 u;
                u.x = bt * (v0.x - wk.x);
                u.y = bt * (v0.y - wk.y);
                u.z = bt * (v1.x - wk.z);
                u.w = bt * (v1.y - wk.w);
#pragma unroll
                for (int m = 0; m < kRowsPerWarp; ++m) fma4(s[m], rowk[t * kD + 8 * m + rsub], u);
                if (o && rsub == 0) {
                    const float qk = s_qk[t];
                    float4 ov;
                    ov.x = scale * fmaf(qk, u.x, wq.x);
                    ov.y = scale * fmaf(qk, u.y, wq.y);
                    ov.z = scale * fmaf(qk, u.z, wq.z);
                    ov.w = scale * fmaf(qk, u.w, wq.w);
                    const size_t orow = ((static_cast<size_t>(b) * T + t) * H + h) * kD;
                    if constexpr (kOutF32) {
                        reinterpret_cast<float4 *>(static_cast<float *>(o) + orow)[4 * warp + cq] = ov;
                    } else {
                        uint2 pk;
                        pk.x = static_cast<uint32_t>(f32_to_bf16(ov.x)) | (static_cast<uint32_t>(f32_to_bf16(ov.y)) << 16);
                        pk.y = static_cast<uint32_t>(f32_to_bf16(ov.z)) | (static_cast<uint32_t>(f32_to_bf16(ov.w)) << 16);
                        reinterpret_cast<uint2 *>(static_cast<uint16_t *>(o) + orow)[4 * warp + cq] = pk;
                    }
                }
            }
        }
        // 7. the new state (the lazy form's rows times their final L)
        if (write_state && n > 0) {
            float4 *dst = reinterpret_cast<float4 *>(S + static_cast<size_t>(bh) * kD * kD) + thread_f4;
            const float4 *rl = rowf + (n - 1) * kD + rsub;
#pragma unroll
            for (int r = 0; r < kRowsPerWarp; ++r) {
                if (lazy) {
                    const float l = rl[8 * r].z;
                    s[r].x *= l;
                    s[r].y *= l;
                    s[r].z *= l;
                    s[r].w *= l;
                }
                __stcs(dst + r * 8 * kVec, s[r]);
            }
        }
        // raw, rowf and the scalars are rewritten next iteration: every thread must be done
        __syncthreads();
        bh = nbh;
        n = nn;
    }
    cp_async_wait_all();
}

}  // namespace

namespace lad {
int take_device_error_kda(cudaStream_t s, int *code) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_kda_error, sizeof v, 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return set_error(LAD_ECUDA, "lad_device_error: %s", cudaGetErrorString(e));
    if (v) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_kda_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return set_error(LAD_ECUDA, "lad_device_error: %s", cudaGetErrorString(e));
    }
    *code = v;
    return LAD_OK;
}
}  // namespace lad

namespace {
// One head per CTA, or two (kPair) when B * H is between one and two times the resident CTAs:
// then every CTA is resident at once and all state bytes are requested together.
// With `overlap` the launch is a programmatic dependent of the kernel before it on the stream (see
// the wait at the top of the kernel).
template <bool kPair, bool kOutF32, bool kFusedConv>
cudaError_t launch_one(unsigned grid, size_t smem, bool overlap, cudaStream_t s, const uint16_t *q, const uint16_t *k,
                       const uint16_t *v, long long stride, const float *alpha, const float *beta, float *S, void *o,
                       int H, float scale, int l2, const ConvIn &cv, const GateIn &gi, int units) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = overlap ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kda_decode_kernel<kOutF32, kFusedConv, kPair>, q, k, v, stride, alpha, beta, S, o,
                              H, scale, l2, cv, gi, units);
}

template <bool kOutF32, bool kFusedConv>
int launch_decode(const char *name, const uint16_t *q, const uint16_t *k, const uint16_t *v, long long stride,
                  const float *alpha, const float *beta, float *S, void *o, int units, int H, float scale, int l2,
                  const ConvIn &cv, const GateIn &gi, bool overlap, cudaStream_t s) {
    const int sms = lad::device_sm_count();
    const long long slots = 2LL * (sms > 0 ? sms : 0);
    if (sms > 0 && units > slots && units <= 2 * slots) {
        static std::mutex mu;
        static bool done[64] = {};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess || dev < 0 || dev >= 64)
            return lad::set_error(LAD_ECUDA, "%s: cudaGetDevice: %s", name, cudaGetErrorString(e));
        {
            std::lock_guard<std::mutex> lock(mu);
            if (!done[dev]) {
                e = cudaFuncSetAttribute(kda_decode_kernel<kOutF32, kFusedConv, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmemBytes);
                if (e != cudaSuccess)
                    return lad::set_error(LAD_ECUDA, "%s: smem attribute: %s", name, cudaGetErrorString(e));
                done[dev] = true;
            }
        }
        const cudaError_t e1 = launch_one<true, kOutF32, kFusedConv>(static_cast<unsigned>(slots), kPairSmemBytes,
                                                                     overlap, s, q, k, v, stride, alpha, beta, S, o,
                                                                     H, scale, l2, cv, gi, units);
        if (e1 != cudaSuccess) return lad::set_error(LAD_ECUDA, "%s: launch: %s", name, cudaGetErrorString(e1));
    } else {
        const cudaError_t e1 = launch_one<false, kOutF32, kFusedConv>(static_cast<unsigned>(units), 0, overlap, s, q,
                                                                      k, v, stride, alpha, beta, S, o, H, scale, l2,
                                                                      cv, gi, units);
        if (e1 != cudaSuccess) return lad::set_error(LAD_ECUDA, "%s: launch: %s", name, cudaGetErrorString(e1));
    }
    return lad::check_launch(name);
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
    if (flags & ~(LAD_FLAG_OUT_FP32 | LAD_FLAG_L2NORM_QK | LAD_FLAG_OVERLAP_PREV))
        return set_error(LAD_EINVAL, "kda_decode_step: unknown flags 0x%x", flags);
    const long long blocks = static_cast<long long>(B) * H;
    if (blocks > 0x7fffffffLL) return set_error(LAD_EUNSUPPORTED, "kda_decode_step: B*H too large");
    const int l2 = (flags & LAD_FLAG_L2NORM_QK) ? 1 : 0;
    cudaStream_t s = lad::as_stream(stream);
    const ConvIn none{nullptr, nullptr, nullptr, nullptr, 0};
    const uint16_t *qq = reinterpret_cast<const uint16_t *>(q), *kk = reinterpret_cast<const uint16_t *>(k),
                   *vv = reinterpret_cast<const uint16_t *>(v);
    const int units = static_cast<int>(blocks);
    const bool ov = (flags & LAD_FLAG_OVERLAP_PREV) != 0;
    return f32 ? launch_decode<true, false>("kda_decode_step", qq, kk, vv, stride, alpha, beta, S, o, units, H, scale,
                                            l2, none, GateIn{}, ov, s)
               : launch_decode<false, false>("kda_decode_step", qq, kk, vv, stride, alpha, beta, S, o, units, H, scale,
                                             l2, none, GateIn{}, ov, s);
}

namespace {
int conv_decode(const char *name, const lad_bf16 *x, lad_bf16 *conv_tail, const lad_bf16 *conv_w,
                const lad_bf16 *conv_bias, const float *alpha, const float *beta, float *S, const GateIn &gi, void *o,
                int B, int H, int dk, int dv, int K, float scale, unsigned flags, void *stream) {
    using lad::set_error;
    if (B < 0 || H < 0) return set_error(LAD_EINVAL, "%s: negative B or H", name);
    if (dk != kD || dv != kD) return set_error(LAD_EUNSUPPORTED, "%s: dk = dv = 128 only", name);
    if (K != 4) return set_error(LAD_EUNSUPPORTED, "%s: K = 4 only", name);
    if (flags & ~(LAD_FLAG_OUT_FP32 | LAD_FLAG_L2NORM_QK | LAD_FLAG_SILU | LAD_FLAG_OVERLAP_PREV))
        return set_error(LAD_EINVAL, "%s: unknown flags 0x%x", name, flags);
    if (B == 0 || H == 0) return LAD_OK;
    if (!x || !conv_tail || !conv_w || !alpha || !beta || !S || !o) return set_error(LAD_EINVAL, "%s: null pointer", name);
    if (!lad::aligned(S, 16) || !lad::aligned(conv_w, 8))
        return set_error(LAD_EUNSUPPORTED, "%s: S 16-byte and conv_w 8-byte aligned", name);
    const bool f32 = (flags & LAD_FLAG_OUT_FP32) != 0;
    if (!lad::aligned(o, f32 ? 16 : 8)) return set_error(LAD_EUNSUPPORTED, "%s: o misaligned", name);
    if (gi.g && (!lad::aligned(gi.g, 8) || (gi.w && !lad::aligned(gi.w, 16))))
        return set_error(LAD_EUNSUPPORTED, "%s: gate 8-byte and norm weight 16-byte aligned", name);
    const long long blocks = static_cast<long long>(B) * H;
    if (blocks > 0x7fffffffLL) return set_error(LAD_EUNSUPPORTED, "%s: B*H too large", name);
    const int l2 = (flags & LAD_FLAG_L2NORM_QK) ? 1 : 0;
    const ConvIn cv{x, conv_tail, conv_w, conv_bias, (flags & LAD_FLAG_SILU) ? 1 : 0};
    cudaStream_t s = lad::as_stream(stream);
    const int units = static_cast<int>(blocks);
    const bool ov = (flags & LAD_FLAG_OVERLAP_PREV) != 0;
    return f32 ? launch_decode<true, true>(name, nullptr, nullptr, nullptr, 0, alpha, beta, S, o, units, H, scale, l2,
                                           cv, gi, ov, s)
               : launch_decode<false, true>(name, nullptr, nullptr, nullptr, 0, alpha, beta, S, o, units, H, scale, l2,
                                            cv, gi, ov, s);
}
}  // namespace

extern "C" int kda_conv_decode_step(const lad_bf16 *x, lad_bf16 *conv_tail, const lad_bf16 *conv_w,
                                    const lad_bf16 *conv_bias, const float *alpha, const float *beta, float *S, void *o,
                                    int B, int H, int dk, int dv, int K, float scale, unsigned flags, void *stream) {
    return conv_decode("kda_conv_decode_step", x, conv_tail, conv_w, conv_bias, alpha, beta, S, GateIn{}, o, B, H, dk,
                       dv, K, scale, flags, stream);
}

extern "C" int kda_conv_decode_step_gated(const lad_bf16 *x, lad_bf16 *conv_tail, const lad_bf16 *conv_w,
                                          const lad_bf16 *conv_bias, const float *alpha, const float *beta, float *S,
                                          const lad_bf16 *gate, const float *norm_w, float eps, void *o, int B, int H,
                                          int dk, int dv, int K, float scale, unsigned flags, void *stream) {
    const char *name = "kda_conv_decode_step_gated";
    if (B > 0 && H > 0 && !gate) return lad::set_error(LAD_EINVAL, "%s: null gate", name);
    if (!(eps >= 0.f) || eps == INFINITY) return lad::set_error(LAD_EINVAL, "%s: eps must be finite and >= 0", name);
    return conv_decode(name, x, conv_tail, conv_w, conv_bias, alpha, beta, S,
                       GateIn{reinterpret_cast<const uint16_t *>(gate), norm_w, eps}, o, B, H, dk, dv, K, scale, flags,
                       stream);
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
    if (!lad::aligned(S, 16) || !lad::aligned(q, 16) || !lad::aligned(k, 16) || !lad::aligned(v, 16) ||
        !lad::aligned(alpha, 16))
        return set_error(LAD_EUNSUPPORTED, "kda_decode_multi: S, q, k, v and alpha must be 16-byte aligned");
    const bool f32 = (flags & LAD_FLAG_OUT_FP32) != 0;
    if (o && !lad::aligned(o, f32 ? 16 : 8)) return set_error(LAD_EUNSUPPORTED, "kda_decode_multi: o misaligned");
    const long long heads = static_cast<long long>(B) * H;
    if (heads > 0x7fffffffLL) return set_error(LAD_EUNSUPPORTED, "kda_decode_multi: B*H too large");
    const int sms = lad::device_sm_count();
    if (sms <= 0) return set_error(LAD_ECUDA, "kda_decode_multi: cannot query the SM count");
    const int grid = static_cast<int>(std::min<long long>(heads, static_cast<long long>(kMultiCtasPerSm) * sms));
    const int smem = multi_smem_bytes(T);
    {
        static std::mutex mu;
        static bool done[64] = {};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess || dev < 0 || dev >= 64)
            return set_error(LAD_ECUDA, "kda_decode_multi: cudaGetDevice: %s", cudaGetErrorString(e));
        std::lock_guard<std::mutex> lock(mu);
        if (!done[dev]) {
            const int mx = multi_smem_bytes(kMaxMultiTokens);
            e = cudaFuncSetAttribute(kda_decode_multi_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(kda_decode_multi_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         mx);
            if (e != cudaSuccess)
                return set_error(LAD_ECUDA, "kda_decode_multi: smem attribute: %s", cudaGetErrorString(e));
            done[dev] = true;
        }
    }
    const int l2 = (flags & LAD_FLAG_L2NORM_QK) ? 1 : 0;
    const int write_state = (flags & LAD_FLAG_KEEP_STATE) ? 0 : 1;
    cudaStream_t s = lad::as_stream(stream);
    if (f32)
        kda_decode_multi_kernel<true><<<grid, kThreads, smem, s>>>(q, k, v, alpha, beta, S, o, n_tokens, B, T, H,
                                                                   scale, l2, write_state);
    else
        kda_decode_multi_kernel<false><<<grid, kThreads, smem, s>>>(q, k, v, alpha, beta, S, o, n_tokens, B, T, H,
                                                                    scale, l2, write_state);
    return lad::check_launch("kda_decode_multi");
}
