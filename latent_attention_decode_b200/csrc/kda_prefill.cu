// KDA chunked prefill on B200: the gated delta rule over T tokens in chunks of 64, in the WY / UT
// form, with every contraction on the tensor cores (tcgen05) and the fp32 state carried in tensor
// memory from chunk to chunk.
//
// Source: "Ling-3.1-flash: a 560B hybrid-attention MoE, counted from its safetensors headers",
// section "How KDA and MLA split the work" (gated delta rule, per-channel decay alpha, per-head
// strength beta, 128x128 state per head). The chunked form is not on the page; it is the
// token-by-token recurrence (S' = Diag(alpha) S; u = beta (v - S'^T k); S = S' + k u^T;
// o = scale S^T q) unrolled over a chunk. Inside a chunk (rows r = tokens, g_r = prod_{s<=r}
// alpha_s per key channel, S0 the state entering the chunk):
//   Kt = K*g, Kh = K/g, Qt = Q*g                                  (elementwise)
//   A  = strict_lower(diag(beta) Kt Kh^T),  T = (I + A)^-1,  Tb = T diag(beta)
//   W  = Tb Kt,  U = Tb V - W S0
//   O  = scale (Qt S0 + lower(Qt Kh^T) U)
//   S  = Diag(g_last) (S0 + Kh^T U)        (= Diag(g_last) S0 + (K * g_last/g)^T U)
//
// Two paths. With a workspace (the fast one), two kernels per segment of up to 128 chunks: the
// prep kernel computes, for every chunk in parallel, the state-independent operands that need the
// CUDA cores (fp16 operands, kind::f16) into a record per chunk, and the chain kernel runs the
// chunk's tensor-core work around the state, one CTA per (sequence, head) (see "Split path"
// below). Without one, a single kernel does both with tf32
// operands; the d_v columns of S are independent, so there a CTA owns one (sequence, head, half
// of d_v) and walks its chunks in order: 128 CTAs for one sequence of 64 heads.
//
// Single kernel, per chunk (two warpgroups; warp 0 issues the MMAs, converged, elect.sync):
//   1. load q, k, alpha, v, beta; running products g; write the operand tiles
//   2. MMA  [Qt; Kt] Kh^T  (M = 128: rows 0-63 give Qt Kh^T, rows 64-127 give Kt Kh^T), and
//           Y = Kt S0 (it needs no T: W S0 = Tb (Kt S0), so W itself is never formed); then
//           O = Qt S0 is issued without waiting, to run during step 3
//   3. lower(Qt Kh^T) -> operand; A -> fp32 scratch; Y -> operand; T = (I + A)^-1 by 16x16
//      blocked forward substitution on the CUDA cores; Tb -> operand
//   4. MMA  U' = Tb V,  X = Tb Y;  U = U' - X -> operand
//   5. MMA  O += lower(Qt Kh^T) U;  S += Kh^T U
//   6. O -> HBM; S <- Diag(g_last) S in TMEM, and -> next chunk's S0 operand (HBM after the last)
// Every operand tile is K-major fp32 with the 128-byte swizzle (tf32 operands read MN-major
// would need a different swizzle; storing the transposes instead keeps one layout): the tiles
// that a contraction needs "the other way round" (Kt^T, Kh^T, V^T / U^T, S0^T) are written
// transposed by the threads that own the data. Values are rounded to tf32 to nearest (cvt.rna)
// when written, so the tensor core's tf32 read loses nothing further. tf32 operands keep every
// output within a few 1e-4 relative of fp64; bf16 operands for the derived matrices would cost
// ~1.6e-3, too close to the 2e-3 output budget. The state master stays fp32 in TMEM.
// Padded rows of a short last chunk get q = k = v = 0, alpha = 1, beta = 0, which makes them
// contribute nothing; their outputs are not stored.
#include <cuda.h>

#include <mutex>

#include "sm100_ptx.cuh"

namespace {

using namespace lad::ptx;
using lad::dev::bf16_to_f32;

constexpr int kC = 64;         // chunk length
constexpr int kDk = 128;       // key width
constexpr int kDv = 128;       // value width
constexpr int kDvh = 64;       // value columns per CTA
constexpr int kThreads = 256;

// Shared memory (bytes). An operand tile is a set of blocks, one per 32 fp32 columns, each block
// holding the tile's rows as 128-byte swizzled rows; "stride" is the distance between blocks.
constexpr uint32_t kOffXQK = 0;        // [Qt; Kt]: 128 rows (tokens) x 128 (d_k), stride 16 KiB
constexpr uint32_t kOffTT = 8192;      //   Tb [64 r][64 s] in the Kt half of XQK blocks 0-1 (stride 16 KiB)
constexpr uint32_t kOffQM = 40960;     //   lower(Qt Kh^T) [64][64] in the Kt half of blocks 2-3
constexpr uint32_t kOffKH = 65536;     // Kh [64 tokens][128 d_k], stride 8 KiB; then A/T scratch; then W
constexpr uint32_t kOffYT = 98304;     // Y^T = (Kt S0)^T [64 d_v][64 tokens], stride 8 KiB
constexpr uint32_t kOffKHT = 131072;   // Kh^T [128 d_k][64 tokens], stride 16 KiB
constexpr uint32_t kOffVT = 163840;    // V^T, then U^T: [64 d_v][64 tokens], stride 8 KiB
constexpr uint32_t kOffSOT = 180224;   // S0^T [64 d_v][128 d_k], stride 8 KiB
constexpr uint32_t kOffMisc = 212992;
constexpr uint32_t kStr16 = 16384, kStr8 = 8192;
constexpr uint32_t kMiscBeta = 0, kMiscRq = 256, kMiscRk = 512, kMiscGc = 768, kMiscBar = 1280, kMiscTmem = 1288,
                   kMiscAbort = 1292, kMiscTmaBar = 1296, kMiscOct = 2048;  // s_oct: [8 octets][128] fp32
// Raw inputs of the next chunk, TMA-staged over tiles that are dead once a chunk's last MMA has
// completed (Y^T, Kh^T and U^T): alpha [64][128] fp32, q and k [64][128] bf16, v [64][64] bf16.
constexpr uint32_t kOffStA = kOffYT;             // 32 KiB
constexpr uint32_t kOffStQ = kOffStA + 32768;    // 16 KiB
constexpr uint32_t kOffStK = kOffStQ + 16384;    // 16 KiB
constexpr uint32_t kOffStV = kOffStK + 16384;    // 8 KiB, ends inside the V^T tile
constexpr uint32_t kStageTx = 32768 + 16384 + 16384 + 8192;
constexpr uint32_t kSmemBytes = kOffMisc + kMiscOct + 8 * 128 * 4 + 1024;  // + alignment slack

// TMEM columns (fp32)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc1 = 0;    // M=128 x 64: [Qt Kh^T ; Kt Kh^T]
constexpr uint32_t kColY = 64;      // M=64 x 64: Y = Kt S0
constexpr uint32_t kColU = 128;     // M=64 x 64: U' = Tb V
constexpr uint32_t kColX = 192;     // M=64 x 64: Tb Y = W S0
constexpr uint32_t kColO = 256;     // M=64 x 64
constexpr uint32_t kColS = 320;     // M=128 x 64: state master (rows d_k)

constexpr uint32_t kIdesc128 = make_idesc(128, 64, kFmtTf32, 0, 0);
constexpr uint32_t kIdesc64 = make_idesc(64, 64, kFmtTf32, 0, 0);

__device__ int g_prefill_error = 0;

struct Args {
    const uint16_t *q, *k, *v;
    const float *alpha, *beta;
    float *S;
    void *o;
    int B, T, H;
    float scale;
    int l2norm, out_f32;
};

__device__ __forceinline__ void st_tile4(uint8_t *tile, int row, int col, uint32_t stride, float a, float b, float c,
                                         float d) {
    *reinterpret_cast<float4 *>(tile + sw128_off32(row, col, stride)) =
        make_float4(round_tf32(a), round_tf32(b), round_tf32(c), round_tf32(d));
}

__device__ __forceinline__ void st_tile1(uint8_t *tile, int row, int col, uint32_t stride, float a) {
    *reinterpret_cast<float *>(tile + sw128_off32(row, col, stride)) = round_tf32(a);
}

// K-major SW128 descriptor of a tile at smem byte `addr` for k-step j (8 tf32 of K per step).
__device__ __forceinline__ uint64_t kdesc(uint64_t base_desc, uint32_t stride, int j) {
    return base_desc + ((static_cast<uint32_t>(j >> 2) * stride + static_cast<uint32_t>(j & 3) * 32u) >> 4);
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int x, int y, int z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

// a tile into L2 only (no shared memory, no barrier; a hint): a later load of it is served from L2
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap *map, int x, int y, int z) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z)
                 : "memory");
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct Maps {
    CUtensorMap q, k, alpha, v;  // 3-D views [B][T][H*128], boxes of 64 tokens
};

// T = (I + A)^-1 for A strictly lower triangular [64][64] (fp32, plain row-major in Apl), by 16x16
// blocks: the diagonal blocks by forward substitution, then M_ik = T_ii A_ik for the six blocks
// below the diagonal in one pass (written over A), then T_ij = -sum_k M_ik T_kj one block row at
// a time. T goes to Tpl (plain) and Tb = T diag(beta) to the operand tile `tt` (stride 16 KiB) as
// each block is final. Called by all kThreads threads; contains block-wide barriers.
__device__ __forceinline__ void solve_tb(float *Apl, float *Tpl, const float *s_beta, uint8_t *tt, int tid) {
    if (tid < kC) {
        const int base = 16 * (tid >> 4), c = tid & 15;
        float t[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            float acc = (rr == c) ? 1.f : 0.f;
#pragma unroll
            for (int ss = 0; ss < rr; ++ss) acc -= Apl[(base + rr) * 64 + base + ss] * t[ss];
            t[rr] = acc;
        }
        const float bc = s_beta[base + c];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            Tpl[(base + rr) * 64 + base + c] = t[rr];
            st_tile1(tt, base + rr, base + c, kStr16, t[rr] * bc);  // Tb = T diag(beta)
        }
    } else {
        // zero the blocks above the diagonal, in T and in the Tb operand: (bi, bj) with bi < bj
        for (int e = tid - kC; e < 6 * 64; e += kThreads - kC) {
            const int blk = e >> 6, rr = (e >> 2) & 15, cc = (e & 3) * 4;
            const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
            const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            *reinterpret_cast<float4 *>(Tpl + (16 * bi + rr) * 64 + 16 * bj + cc) = make_float4(0.f, 0.f, 0.f, 0.f);
            st_tile4(tt, 16 * bi + rr, 16 * bj + cc, kStr16, 0.f, 0.f, 0.f, 0.f);
        }
    }
    __syncthreads();
    // Off-diagonal blocks: T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj = -sum_k M_ik T_kj with
    // M_ik = T_ii A_ik, which needs only the diagonal blocks: all six M blocks in one pass (kept in
    // A's place), then one pass per block row. A thread computes 1x4 strips (row rr, columns cc).
    {
        // M_ik for (i, k) = (1,0), (2,0), (2,1), (3,0), (3,1), (3,2): 6 blocks x 64 strips
        float4 m[2];
        int mi[2], mk[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = tid + h * kThreads;
            m[h] = make_float4(0.f, 0.f, 0.f, 0.f);
            mi[h] = -1;
            if (e < 6 * 64) {
                const int blk = e >> 6, rr = (e >> 2) & 15, cc = (e & 3) * 4;
                const int i = blk == 0 ? 1 : (blk < 3 ? 2 : 3);
                const int k = blk == 0 ? 0 : (blk < 3 ? blk - 1 : blk - 3);
                mi[h] = i;
                mk[h] = k;
#pragma unroll
                for (int ss = 0; ss < 16; ++ss) {
                    const float t = Tpl[(16 * i + rr) * 64 + 16 * i + ss];
                    const float4 a4 = *reinterpret_cast<const float4 *>(Apl + (16 * i + ss) * 64 + 16 * k + cc);
                    m[h].x = fmaf(t, a4.x, m[h].x);
                    m[h].y = fmaf(t, a4.y, m[h].y);
                    m[h].z = fmaf(t, a4.z, m[h].z);
                    m[h].w = fmaf(t, a4.w, m[h].w);
                }
            }
        }
        __syncthreads();  // every read of A is done: the M blocks replace it
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = tid + h * kThreads;
            if (mi[h] >= 0) {
                const int rr = (e >> 2) & 15, cc = (e & 3) * 4;
                *reinterpret_cast<float4 *>(Apl + (16 * mi[h] + rr) * 64 + 16 * mk[h] + cc) = m[h];
            }
        }
        __syncthreads();
    }
#pragma unroll 1
    for (int bi = 1; bi < 4; ++bi) {
        // block row bi: blocks bj < bi, one strip per thread (bi * 64 threads)
        if (tid < bi * 64) {
            const int bj = tid >> 6, rr = (tid >> 2) & 15, cc = (tid & 3) * 4;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int kb = bj; kb < bi; ++kb) {
#pragma unroll
                for (int ss = 0; ss < 16; ++ss) {
                    const float a = Apl[(16 * bi + rr) * 64 + 16 * kb + ss];
                    const float4 t4 = *reinterpret_cast<const float4 *>(Tpl + (16 * kb + ss) * 64 + 16 * bj + cc);
                    acc.x = fmaf(a, t4.x, acc.x);
                    acc.y = fmaf(a, t4.y, acc.y);
                    acc.z = fmaf(a, t4.z, acc.z);
                    acc.w = fmaf(a, t4.w, acc.w);
                }
            }
            *reinterpret_cast<float4 *>(Tpl + (16 * bi + rr) * 64 + 16 * bj + cc) =
                make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
            const int c = 16 * bj + cc;
            st_tile4(tt, 16 * bi + rr, c, kStr16, -acc.x * s_beta[c], -acc.y * s_beta[c + 1],
                     -acc.z * s_beta[c + 2], -acc.w * s_beta[c + 3]);
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kThreads, 1) kda_prefill_kernel(Args p, const __grid_constant__ Maps maps) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    float *s_beta = reinterpret_cast<float *>(sm + kOffMisc + kMiscBeta);
    float *s_rq = reinterpret_cast<float *>(sm + kOffMisc + kMiscRq);
    float *s_rk = reinterpret_cast<float *>(sm + kOffMisc + kMiscRk);
    float *s_gc = reinterpret_cast<float *>(sm + kOffMisc + kMiscGc);
    float *s_oct = reinterpret_cast<float *>(sm + kOffMisc + kMiscOct);
    const uint32_t bar = sbase + kOffMisc + kMiscBar;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc + kMiscTmem);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + kMiscAbort);
    const uint32_t tma_bar = sbase + kOffMisc + kMiscTmaBar;
    float *Apl = reinterpret_cast<float *>(sm + kOffKH);  // [64][64] fp32, plain row-major
    float *Tpl = reinterpret_cast<float *>(sm + kOffKH + 64 * 64 * 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // TMEM: warp w reads sub-partition w % 4; warps w and w + 4 split a 64-column accumulator
    // into column halves.
    const int sp = warp & 3, cg = warp >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(32 * sp) << 16;
    const int row128 = 32 * sp + lane;  // row of an M = 128 accumulator held by this thread
    const int row64 = 16 * sp + lane;   // row of an M = 64 accumulator (lanes 0-15 hold rows)
    const int half = blockIdx.x & 1;
    const int bh = blockIdx.x >> 1;
    const int b = bh / p.H, h = bh - b * p.H;
    const uint64_t d0 = smem_desc(sbase, 16, 1024, kLayoutSw128);  // K-major SW128 at smem offset 0

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(tma_bar, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t phase = 0;
    bool ok = true;

    auto mma_sync = [&](auto &&issue) {
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            tc_fence_after();
            issue();
            tc_commit(bar);
        }
        const bool w = wait_bar(bar, phase, abort_flag, &g_prefill_error, lad::kErrPrefill);
        phase ^= 1;
        tc_fence_after();
        return __syncthreads_and(w) != 0;
    };

    // ---- initial state: TMEM master row = key channel, S0^T column; 32 value columns per thread ----
    {
        const float *S0 = p.S + (static_cast<size_t>(bh) * kDk + row128) * kDv + half * kDvh + 32 * cg;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(S0 + j);
            v[j] = x.x;
            v[j + 1] = x.y;
            v[j + 2] = x.z;
            v[j + 3] = x.w;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) st_tile1(sm + kOffSOT, 32 * cg + j, row128, kStr8, v[j]);
        tmem_st32(tmem + lane_base + kColS + 32 * cg, v);
        tmem_wait_st();
    }

    // the next chunk's raw inputs, staged by TMA (thread 0); rows past T read as zeros
    // One barrier phase per chunk's staging, expecting all its bytes at once: alpha (over Y^T, dead
    // once step 4's MMAs are complete) goes first, q, k and v (over Kh^T and U^T) after step 5.
    auto stage_alpha = [&](int chunk) {
        fence_async_smem();
        mbar_arrive_tx_raw(tma_bar, kStageTx);
        tma_load_3d(sbase + kOffStA, &maps.alpha, h * kDk, chunk * kC, b, tma_bar);
    };
    auto stage_qkv = [&](int chunk) {
        fence_async_smem();
        const int t = chunk * kC;
        tma_load_3d(sbase + kOffStQ, &maps.q, h * kDk, t, b, tma_bar);
        tma_load_3d(sbase + kOffStK, &maps.k, h * kDk, t, b, tma_bar);
        tma_load_3d(sbase + kOffStV, &maps.v, h * kDv + half * kDvh, t, b, tma_bar);
    };
    auto stage = [&](int chunk) {
        stage_alpha(chunk);
        stage_qkv(chunk);
    };
    int qkv_owed = -1;  // a chunk whose alpha is staged but whose q, k, v are not yet
    uint32_t tma_phase = 0;
    int pending = 0;  // a staging copy is in flight
    const int nchunks = (p.T + kC - 1) / kC;
    if (tid == 0) stage(0);
    pending = 1;
    for (int ch = 0; ch < nchunks && ok; ++ch) {
        const int t0 = ch * kC;
        const int n = min(kC, p.T - t0);
        const size_t tok0 = (static_cast<size_t>(b) * p.T + t0) * p.H + h;  // token row of (b, t0, h)
        const size_t tstride = static_cast<size_t>(p.H);                      // rows between tokens

        // ---- 1a. beta, the staged raw inputs, per-token inverse norms (L2 flag) ----
        if (tid < kC) s_beta[tid] = (tid < n) ? p.beta[tok0 + tid * tstride] : 0.f;
        {
            const bool w = wait_bar(tma_bar, tma_phase, abort_flag, &g_prefill_error, lad::kErrPrefill);
            tma_phase ^= 1;
            pending = 0;
            ok = __syncthreads_and(w) != 0;
            if (!ok) break;
        }
        if (p.l2norm) {
            const uint16_t *sq = reinterpret_cast<const uint16_t *>(sm + kOffStQ);
            const uint16_t *sk = reinterpret_cast<const uint16_t *>(sm + kOffStK);
#pragma unroll 1
            for (int r = warp; r < kC; r += kThreads / 32) {
                const uint2 qw = *reinterpret_cast<const uint2 *>(sq + r * kDk + 4 * lane);
                const uint2 kw = *reinterpret_cast<const uint2 *>(sk + r * kDk + 4 * lane);
                const float2 q0 = lad::dev::bf16x2_to_f32(qw.x), q1 = lad::dev::bf16x2_to_f32(qw.y);
                const float2 k0 = lad::dev::bf16x2_to_f32(kw.x), k1 = lad::dev::bf16x2_to_f32(kw.y);
                float sqs = q0.x * q0.x + q0.y * q0.y + q1.x * q1.x + q1.y * q1.y;
                float sks = k0.x * k0.x + k0.y * k0.y + k1.x * k1.x + k1.y * k1.y;
#pragma unroll
                for (int o = 16; o; o >>= 1) {
                    sqs += __shfl_xor_sync(0xffffffffu, sqs, o);
                    sks += __shfl_xor_sync(0xffffffffu, sks, o);
                }
                if (lane == 0) {
                    s_rq[r] = rsqrtf(sqs + 1e-6f);
                    s_rk[r] = rsqrtf(sks + 1e-6f);
                }
            }
        } else if (tid < kC) {
            s_rq[tid] = 1.f;
            s_rk[tid] = 1.f;
        }
        __syncthreads();

        // ---- 1b. running decay and the operand tiles. Warp w takes tokens 8w .. 8w+7 and lane l
        //          the key channels 4l .. 4l+3 (one 512-byte row segment per warp access); the
        //          product over earlier token octets comes through shared memory ----
        {
            const int o = warp, c4 = 4 * lane;
            const float *sa = reinterpret_cast<const float *>(sm + kOffStA);
            const uint16_t *sq = reinterpret_cast<const uint16_t *>(sm + kOffStQ);
            const uint16_t *sk = reinterpret_cast<const uint16_t *>(sm + kOffStK);
            float4 gl[8];  // running product within the octet
            float4 run = make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int r = 8 * o + u;
                const float4 a = (r < n) ? *reinterpret_cast<const float4 *>(sa + r * kDk + c4)
                                         : make_float4(1.f, 1.f, 1.f, 1.f);
                run.x *= a.x;
                run.y *= a.y;
                run.z *= a.z;
                run.w *= a.w;
                gl[u] = run;
            }
            *reinterpret_cast<float4 *>(s_oct + o * kDk + c4) = run;
            __syncthreads();
            float4 excl = make_float4(1.f, 1.f, 1.f, 1.f);  // product over the octets before o
            for (int oo = 0; oo < o; ++oo) {
                const float4 y = *reinterpret_cast<const float4 *>(s_oct + oo * kDk + c4);
                excl.x *= y.x;
                excl.y *= y.y;
                excl.z *= y.z;
                excl.w *= y.w;
            }
            if (o == kThreads / 32 - 1)
                *reinterpret_cast<float4 *>(s_gc + c4) =
                    make_float4(excl.x * run.x, excl.y * run.y, excl.z * run.z, excl.w * run.w);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int r = 8 * o + u;
                const float gg[4] = {excl.x * gl[u].x, excl.y * gl[u].y, excl.z * gl[u].z, excl.w * gl[u].w};
                const uint2 qw = *reinterpret_cast<const uint2 *>(sq + r * kDk + c4);
                const uint2 kw = *reinterpret_cast<const uint2 *>(sk + r * kDk + c4);
                const float2 q0 = lad::dev::bf16x2_to_f32(qw.x), q1 = lad::dev::bf16x2_to_f32(qw.y);
                const float2 k0 = lad::dev::bf16x2_to_f32(kw.x), k1 = lad::dev::bf16x2_to_f32(kw.y);
                const float rq = s_rq[r], rk = s_rk[r];
                const float qv[4] = {q0.x * rq, q0.y * rq, q1.x * rq, q1.y * rq};
                const float kv[4] = {k0.x * rk, k0.y * rk, k1.x * rk, k1.y * rk};
                st_tile4(sm + kOffXQK, r, c4, kStr16, qv[0] * gg[0], qv[1] * gg[1], qv[2] * gg[2], qv[3] * gg[3]);
                st_tile4(sm + kOffXQK, kC + r, c4, kStr16, kv[0] * gg[0], kv[1] * gg[1], kv[2] * gg[2], kv[3] * gg[3]);
                st_tile4(sm + kOffKH, r, c4, kStr8, __fdividef(kv[0], gg[0]), __fdividef(kv[1], gg[1]),
                         __fdividef(kv[2], gg[2]), __fdividef(kv[3], gg[3]));
            }
            // V^T: thread -> value column j = tid % 64, tokens 16 * (tid / 64) .. + 15
            const uint16_t *sv = reinterpret_cast<const uint16_t *>(sm + kOffStV);
            const int j = tid & 63, r0 = 16 * (tid >> 6);
            float vv[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) vv[r] = bf16_to_f32(sv[(r0 + r) * kDvh + j]);
            __syncthreads();  // the staging area is read; Kh^T and V^T overwrite it
#pragma unroll
            for (int r = 0; r < 16; r += 4) st_tile4(sm + kOffVT, j, r0 + r, kStr8, vv[r], vv[r + 1], vv[r + 2], vv[r + 3]);
            // Kh^T: thread -> channel i (row), tokens of half th, from the tile above
            const int i = tid & (kDk - 1), th = tid >> 7;
#pragma unroll 4
            for (int r = (kC / 2) * th; r < (kC / 2) * (th + 1); r += 4) {
                float kh[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    kh[u] = *reinterpret_cast<const float *>(sm + kOffKH + sw128_off32(r + u, i, kStr8));
                st_tile4(sm + kOffKHT, i, r, kStr16, kh[0], kh[1], kh[2], kh[3]);
            }
        }

        // ---- 2. [Qt; Kt] Kh^T and Y = Kt S0 (Kt: rows 64-127 of the [Qt; Kt] tile) ----
        ok = mma_sync([&] {
#pragma unroll
            for (int j = 0; j < kDk / 8; ++j) {
                const uint64_t sot = kdesc(d0 + (kOffSOT >> 4), kStr8, j);
                tc_mma_tf32(tmem + kColAcc1, kdesc(d0 + (kOffXQK >> 4), kStr16, j), kdesc(d0 + (kOffKH >> 4), kStr8, j),
                            kIdesc128, j > 0);
                tc_mma_tf32(tmem + kColY, kdesc(d0 + ((kOffXQK + kC * 128) >> 4), kStr16, j), sot, kIdesc64, j > 0);
            }
        });
        if (!ok) break;
        // O = Qt S0 needs nothing of this chunk's solve and Qt and S0^T stay put until the chunk ends:
        // issued now, it runs while the CUDA cores solve; the commit after step 5's MMAs covers it
        if (warp == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < kDk / 8; ++j)
                tc_mma_tf32(tmem + kColO, kdesc(d0 + (kOffXQK >> 4), kStr16, j), kdesc(d0 + (kOffSOT >> 4), kStr8, j),
                            kIdesc64, j > 0);
        }

        // ---- 3a. lower(Qt Kh^T) -> QM (rows 0-63); A = strict_lower(diag(beta) Kt Kh^T) -> fp32
        //          scratch (rows 64-127); each thread has 32 of the 64 columns of its row ----
        {
            float x[32];
            tmem_ld32(tmem + lane_base + kColAcc1 + 32 * cg, x);
            tmem_wait_ld();
            const int c0 = 32 * cg;
            if (row128 < kC) {
                const int r = row128;
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    st_tile4(sm + kOffQM, r, c0 + j, kStr16, c0 + j <= r ? x[j] : 0.f, c0 + j + 1 <= r ? x[j + 1] : 0.f,
                             c0 + j + 2 <= r ? x[j + 2] : 0.f, c0 + j + 3 <= r ? x[j + 3] : 0.f);
            } else {
                const int r = row128 - kC;
                const float br = s_beta[r];
                float4 *dst = reinterpret_cast<float4 *>(Apl + r * 64 + c0);
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    dst[j / 4] = make_float4(c0 + j < r ? br * x[j] : 0.f, c0 + j + 1 < r ? br * x[j + 1] : 0.f,
                                             c0 + j + 2 < r ? br * x[j + 2] : 0.f, c0 + j + 3 < r ? br * x[j + 3] : 0.f);
            }
            // Y [token][d_v] (M = 64 rows: lanes 0-15) -> Y^T operand
            float y[32];
            tmem_ld32(tmem + lane_base + kColY + 32 * cg, y);
            tmem_wait_ld();
            if (lane < 16) {
#pragma unroll
                for (int j = 0; j < 32; ++j) st_tile1(sm + kOffYT, 32 * cg + j, row64, kStr8, y[j]);
            }
        }
        __syncthreads();

        // ---- 3b. T = (I + A)^-1 and Tb = T diag(beta) -> operand ----
        solve_tb(Apl, Tpl, s_beta, sm + kOffTT, tid);
        // ---- 4. U' = Tb V (B = V^T),  X = Tb Y (B = Y^T);  U = U' - X -> U^T operand ----
        ok = mma_sync([&] {
#pragma unroll
            for (int j = 0; j < kC / 8; ++j) {
                const uint64_t tt = kdesc(d0 + (kOffTT >> 4), kStr16, j);
                tc_mma_tf32(tmem + kColU, tt, kdesc(d0 + (kOffVT >> 4), kStr8, j), kIdesc64, j > 0);
                tc_mma_tf32(tmem + kColX, tt, kdesc(d0 + (kOffYT >> 4), kStr8, j), kIdesc64, j > 0);
            }
        });
        if (!ok) break;
        if (ch + 1 < nchunks) {  // Y^T is dead now: the next chunk's alpha can come in
            if (tid == 0) stage_alpha(ch + 1);
            pending = 1;
            qkv_owed = ch + 1;
        }
        {
            float u[32], x[32];
            tmem_ld32(tmem + lane_base + kColU + 32 * cg, u);
            tmem_ld32(tmem + lane_base + kColX + 32 * cg, x);
            tmem_wait_ld();
            if (lane < 16) {
#pragma unroll
                for (int j = 0; j < 32; ++j) st_tile1(sm + kOffVT, 32 * cg + j, row64, kStr8, u[j] - x[j]);
            }
        }

        // ---- 5. O += lower(Qt Kh^T) U;  S += Kh^T U ----
        ok = mma_sync([&] {
#pragma unroll
            for (int j = 0; j < kC / 8; ++j) {
                const uint64_t ut = kdesc(d0 + (kOffVT >> 4), kStr8, j);
                tc_mma_tf32(tmem + kColO, kdesc(d0 + (kOffQM >> 4), kStr16, j), ut, kIdesc64, 1);
                tc_mma_tf32(tmem + kColS, kdesc(d0 + (kOffKHT >> 4), kStr16, j), ut, kIdesc128, 1);
            }
        });
        if (!ok) break;

        // ---- 6. O -> HBM; S <- Diag(g_last) S (TMEM), S^T -> operand (HBM after the last chunk) ----
        if (qkv_owed >= 0) {  // Kh^T and U^T are dead now
            if (tid == 0) stage_qkv(qkv_owed);
            qkv_owed = -1;
        }
        {
            float ov[32];
            tmem_ld32(tmem + lane_base + kColO + 32 * cg, ov);
            tmem_wait_ld();
            if (lane < 16 && row64 < n) {
                const size_t orow = (tok0 + row64 * tstride) * kDv + half * kDvh + 32 * cg;
                if (p.out_f32) {
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.o) + orow);
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        dst[j / 4] = make_float4(p.scale * ov[j], p.scale * ov[j + 1], p.scale * ov[j + 2],
                                                 p.scale * ov[j + 3]);
                } else {
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.o) + orow);
#pragma unroll
                    for (int j = 0; j < 32; j += 8)
                        dst[j / 8] = make_uint4(lad::dev::f32x2_to_bf16x2(p.scale * ov[j], p.scale * ov[j + 1]),
                                                lad::dev::f32x2_to_bf16x2(p.scale * ov[j + 2], p.scale * ov[j + 3]),
                                                lad::dev::f32x2_to_bf16x2(p.scale * ov[j + 4], p.scale * ov[j + 5]),
                                                lad::dev::f32x2_to_bf16x2(p.scale * ov[j + 6], p.scale * ov[j + 7]));
                }
            }
            const float gc = s_gc[row128];
            float sv[32];
            tmem_ld32(tmem + lane_base + kColS + 32 * cg, sv);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                sv[j] *= gc;
                st_tile1(sm + kOffSOT, 32 * cg + j, row128, kStr8, sv[j]);
            }
            tmem_st32(tmem + lane_base + kColS + 32 * cg, sv);
            if (ch == nchunks - 1) {
                float *Sout = p.S + (static_cast<size_t>(bh) * kDk + row128) * kDv + half * kDvh + 32 * cg;
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(Sout + j) = make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
    }

    // drain: a staging copy still in flight (after an abort) lands, and every MMA this CTA
    // issued completes, before shared memory and TMEM are released
    if (tid == 0 && qkv_owed >= 0) stage_qkv(qkv_owed);  // the phase expects those bytes too
    if (tid == 0 && pending) {
        const uint64_t t0 = lad::dev::globaltimer_ns();
        while (!mbar_try_wait(tma_bar, tma_phase) && lad::dev::globaltimer_ns() - t0 < lad::dev::kWaitLimitNs) {
        }
    }
    if (warp == 0) {
        tc_commit(bar);
        const uint64_t t0 = lad::dev::globaltimer_ns();
        while (!mbar_try_wait(bar, phase) && lad::dev::globaltimer_ns() - t0 < lad::dev::kWaitLimitNs) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}


// ------------------------------------------------------------------------------------------
// Split path (a workspace is given): the chunk-local, state-independent part of every chunk in
// parallel (prep), then the state chain alone (chain), segment by segment. With S0 the state
// entering a chunk, Tb = (I + A)^-1 diag(beta), W = Tb Kt and P = lower(Qt Kh^T), the chunk form is
//   U' = Tb V,  X = W S0,  U = U' - X,  O = scale (Qt S0 + P U),  S = Diag(g_last) (S0 + Kh^T U)
// (the last is Diag(g_last) S0 + (K * g_last / g)^T U with the chunk's decay taken out of the key).
// The prep computes what needs the CUDA cores (the decays, the operand tiles, the triangular
// inverse) and one tensor-core product, W; it writes Qt, W, Kh, P, Tb (as a bf16 hi + lo pair)
// and g_last as one record per chunk. The chain holds S^T (rows d_v, columns d_k) as an fp32
// master in tensor memory and per chunk runs two tensor-core batches (M = 128 value rows), with
// one pass through the threads between them and one after:
//   X^T = S0^T W^T,  O^T = S0^T Qt^T,  U'^T = V^T (Tb_hi + Tb_lo)^T      (V by TMA from the input)
//   U^T = U'^T - X^T  (threads: fp32 -> fp16 operand)
//   S^T += U^T Kh,  O^T += U^T P^T
//   S^T <- S^T Diag(g_last) (threads, fp32), and its fp16 copy (the next chunk's S0^T)
// The decay itself is never rounded to fp16.
// Every operand is fp16 (kind::f16, fp32 accumulation): its rounding unit is that of tf32 and it
// runs at twice tf32's rate with half the bytes; each tile is stored once, rows as formed, and
// the tensor cores read it K-major or MN-major as a contraction needs (no transposed copies).
// U' is formed from the bf16 values with Tb split into bf16 hi + lo (two MMAs): V enters exactly
// as given. Values whose magnitude leaves the fp16 range (65504) would overflow: with unit-norm
// keys that needs a chunk's decay product below about 1.5e-5.
// ------------------------------------------------------------------------------------------

// Record of one (sequence, head, chunk) in the workspace: the chain's operand tiles (fp16 / bf16,
// SW128) and g_last, laid out exactly as in the chain's shared memory (one bulk copy).
constexpr uint32_t kRWQ = 0;           // [W; Qt] [128 rows: 64 W, 64 Qt tok][128 d_k], K-major: 2 blocks x 16 KiB
constexpr uint32_t kRKH = 32768;       // Kh [64 tok][128 d_k]: 2 blocks x 8 KiB (read MN-major)
constexpr uint32_t kRP = 49152;        // P [64 r][64 s], K-major: 8 KiB
constexpr uint32_t kRTH = 57344;       // Tb, bf16 high part [64 r][64 s], K-major: 8 KiB
constexpr uint32_t kRTL = 65536;       // Tb, bf16 low part (Tb - hi): 8 KiB
constexpr uint32_t kRG = 73728;        // g_last [128] fp32
constexpr uint32_t kRecBytes = 74240;  // 580 lines of 128 bytes
#ifndef LAD_PREFILL_SEG_CHUNKS
#define LAD_PREFILL_SEG_CHUNKS 128
#endif
constexpr int kSegChunks = LAD_PREFILL_SEG_CHUNKS;  // chunks per segment (prep, then chain)

// fp16 / bf16 SW128 tiles: 64 two-byte columns per 128-byte row, blocks of 64 columns
__device__ __forceinline__ uint32_t sw128_off16(int row, int col, uint32_t block_bytes) {
    const int cc = col & 63;
    return static_cast<uint32_t>(col >> 6) * block_bytes + static_cast<uint32_t>(row) * 128u +
           static_cast<uint32_t>(((cc >> 3) ^ (row & 7)) << 4) + static_cast<uint32_t>((cc & 7) << 1);
}

// K-major SW128 descriptor of a 16-bit tile for k-step j (16 elements of K per MMA)
__device__ __forceinline__ uint64_t kdesc16(uint64_t base_desc, uint32_t block_bytes, int j) {
    return base_desc + ((static_cast<uint32_t>(j >> 2) * block_bytes + static_cast<uint32_t>(j & 3) * 32u) >> 4);
}

// two floats to a bf16 pair (lo in the low half), rounded to nearest even, in one conversion
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

constexpr uint32_t kIdescA = make_idesc(128, 64, kFmtF16, 0, 0);     // [Kt; Qt] Kh^T
constexpr uint32_t kIdescW = make_idesc(64, 128, kFmtF16, 0, 1);     // W = Tb Kt (Kt read MN-major)
constexpr uint32_t kIdescU = make_idesc(128, 64, kFmtBf16, 1, 0);    // U'^T = V^T Tb^T (V read MN-major)
constexpr uint32_t kIdescSU = make_idesc(128, 128, kFmtF16, 0, 1);   // S^T += U^T Kh (Kh read MN-major)
constexpr uint32_t kIdescXO = make_idesc(128, 128, kFmtF16, 0, 0);  // [X^T | O^T] = S0^T [W; Qt]^T
constexpr uint32_t kIdescO = make_idesc(128, 64, kFmtF16, 0, 0);     // O^T += U^T P^T

struct PrepArgs {
    const float *beta;
    uint8_t *ws;   // this segment's records, [B*H][nseg]
    int *counter;  // the segment's item counter (zero at launch)
    int B, T, H;
    int c0, nseg;  // the segment: chunks c0 .. c0 + nseg - 1
    int l2norm;
};

struct PrepMaps {
    CUtensorMap q, k, alpha;  // 3-D [B][T][H*128], boxes of 128 channels x 64 tokens, no swizzle
};

constexpr int kAS = 68;             // row stride (floats) of the A / T scratch (68: fewer bank conflicts)
constexpr int kPThreads = 512;      // the prep's 16 warps
constexpr uint32_t kPStageTx = 16384 + 16384 + 32768;  // q, k, alpha of an item

// element (r, s) of the three Tb tiles, four consecutive s at once (s % 4 == 0)
__device__ __forceinline__ void put_tb4(uint8_t *tb16, uint8_t *tbh, uint8_t *tbl, int r, int s, float2 ab, float2 cd) {
    const uint32_t off = sw128_off16(r, s, 8192);
    *reinterpret_cast<uint2 *>(tb16 + off) = make_uint2(f32x2_to_f16x2(ab.x, ab.y), f32x2_to_f16x2(cd.x, cd.y));
    const uint32_t h0 = bf16x2_rn(ab.x, ab.y), h1 = bf16x2_rn(cd.x, cd.y);
    *reinterpret_cast<uint2 *>(tbh + off) = make_uint2(h0, h1);
    const float2 la = sub2(ab, lad::dev::bf16x2_to_f32(h0)), lc = sub2(cd, lad::dev::bf16x2_to_f32(h1));
    *reinterpret_cast<uint2 *>(tbl + off) = make_uint2(bf16x2_rn(la.x, la.y), bf16x2_rn(lc.x, lc.y));
}
// T times beta, four columns: the element products of put_tb4's arguments
__device__ __forceinline__ void put_tb4_scaled(uint8_t *tb16, uint8_t *tbh, uint8_t *tbl, int r, int s, float4 t,
                                               float4 b) {
    put_tb4(tb16, tbh, tbl, r, s, mul2(make_float2(t.x, t.y), make_float2(b.x, b.y)),
            mul2(make_float2(t.z, t.w), make_float2(b.z, b.w)));
}


// T = (I + A)^-1 for A strictly lower triangular [64][64] (fp32, row stride kAS), by recursive
// doubling over 16x16 blocks, and Tb = T diag(beta) into the three operand tiles (fp16, and the
// bf16 hi / lo split):
//   (0) the four diagonal blocks by forward substitution, one thread per column;
//   (1) in each 32x32 diagonal block, T_{2p+1,2p} = -T_{2p+1,2p+1} A_{2p+1,2p} T_{2p,2p};
//   (2) the lower-left 32x32 block, -T_hi A_{hi,lo} T_lo.
// The products A T of (1) and (2) are parked in A's upper triangle, which holds no data; the blocks
// of T above its diagonal blocks are zeroed in (1), so that (2) runs over whole 32x32 blocks. Steps
// (1) and (2) run on the group's warps 0-3 (a row, or a row pair, and four columns a thread); in (2)
// its other warps write the rows of Tb that are final already. Called by all kTh threads of a group
// (tid: the thread's index in it), with `sync` that group's barrier. tbh / tbl may point to global
// memory (the record) rather than shared memory: the stores are generic.
template <int kTh, typename Sync>
__device__ __forceinline__ void solve_tb(float *sA, float *sT, const float *s_beta, uint8_t *tb16, uint8_t *tbh,
                                         uint8_t *tbl, int tid, Sync sync) {
    static_assert(kTh > 128 && kTh % 32 == 0, "the solve needs warps beyond the first four");
    const int warp = tid >> 5, lane = tid & 31;
    if (tid < kC) {
        // column c of (I + A_ii)^-1: t_r = [r == c] - sum_{s < r} A_rs t_s (t_s = 0 for s < c); a
        // row of the block comes in four 16-byte loads, and two partial sums halve the FMA chain
        const int i0 = 16 * (tid >> 4), c = tid & 15;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const float4 *arow = reinterpret_cast<const float4 *>(sA + (i0 + r) * kAS + i0);
            float2 acc = make_float2(0.f, 0.f);  // the two partial sums, as one packed pair
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                if (4 * q4 + 3 < r) {
                    const float4 a = arow[q4];
                    acc = fma2(make_float2(a.x, a.y), make_float2(t[4 * q4], t[4 * q4 + 1]), acc);
                    acc = fma2(make_float2(a.z, a.w), make_float2(t[4 * q4 + 2], t[4 * q4 + 3]), acc);
                } else if (4 * q4 < r) {
                    const float4 a = arow[q4];
                    acc.x = fmaf(a.x, t[4 * q4], acc.x);
                    if (4 * q4 + 1 < r) acc.y = fmaf(a.y, t[4 * q4 + 1], acc.y);
                    if (4 * q4 + 2 < r) acc.x = fmaf(a.z, t[4 * q4 + 2], acc.x);
                }
            }
            t[r] = r < c ? 0.f : (r == c ? 1.f : -(acc.x + acc.y));
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) sT[(i0 + r) * kAS + i0 + c] = t[r];  // zeros above the diagonal too
    }
    sync();
    // (1a) Y_p = A_{2p+1,2p} T_{2p,2p} into A at rows 32p .. 32p+15, columns 32p+16 .. 32p+31
    const int q0 = 32 * (warp >> 1), rr = 8 * (warp & 1) + (lane >> 2), cc = 4 * (lane & 3);
    if (warp < 4) {
        float2 acc01 = make_float2(0.f, 0.f), acc23 = acc01;
#pragma unroll
        for (int s2 = 0; s2 < 16; ++s2) {
            const float a = sA[(q0 + 16 + rr) * kAS + q0 + s2];
            const float4 t = *reinterpret_cast<const float4 *>(sT + (q0 + s2) * kAS + q0 + cc);
            acc01 = fma2(make_float2(a, a), make_float2(t.x, t.y), acc01);
            acc23 = fma2(make_float2(a, a), make_float2(t.z, t.w), acc23);
        }
        *reinterpret_cast<float4 *>(sA + (q0 + rr) * kAS + q0 + 16 + cc) = make_float4(acc01.x, acc01.y, acc23.x, acc23.y);
    }
    sync();
    // (1b) T_{2p+1,2p} = -T_{2p+1,2p+1} Y_p; T_{2p,2p+1} = 0
    if (warp < 4) {
        float2 acc01 = make_float2(0.f, 0.f), acc23 = acc01;
#pragma unroll
        for (int s2 = 0; s2 < 16; ++s2) {
            const float t = sT[(q0 + 16 + rr) * kAS + q0 + 16 + s2];
            const float4 y = *reinterpret_cast<const float4 *>(sA + (q0 + s2) * kAS + q0 + 16 + cc);
            acc01 = fma2(make_float2(t, t), make_float2(y.x, y.y), acc01);
            acc23 = fma2(make_float2(t, t), make_float2(y.z, y.w), acc23);
        }
        *reinterpret_cast<float4 *>(sT + (q0 + 16 + rr) * kAS + q0 + cc) =
            make_float4(-acc01.x, -acc01.y, -acc23.x, -acc23.y);
        *reinterpret_cast<float4 *>(sT + (q0 + rr) * kAS + q0 + 16 + cc) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    sync();
    // thread (warps 0-3) of steps (2a) / (2b): rows r2, r2 + 1 of a 32-row block, columns c2 .. c2 + 3
    const int r2 = 2 * (tid >> 3), c2 = 4 * (tid & 7);
    // (2a) R = A_{hi,lo} T_lo into A at rows 0 .. 31, columns 32 .. 63. Warps 4-15: Tb rows 0-31
    //      (T_lo times beta; zero right of column 31)
    if (warp < 4) {
        float2 a00 = make_float2(0.f, 0.f), a01 = a00, a10 = a00, a11 = a00;  // row, column pair
#pragma unroll 8
        for (int s = 0; s < 32; ++s) {
            const float x0 = sA[(32 + r2) * kAS + s], x1 = sA[(33 + r2) * kAS + s];
            const float4 t = *reinterpret_cast<const float4 *>(sT + s * kAS + c2);
            const float2 tlo = make_float2(t.x, t.y), thi = make_float2(t.z, t.w);
            a00 = fma2(make_float2(x0, x0), tlo, a00);
            a01 = fma2(make_float2(x0, x0), thi, a01);
            a10 = fma2(make_float2(x1, x1), tlo, a10);
            a11 = fma2(make_float2(x1, x1), thi, a11);
        }
        *reinterpret_cast<float4 *>(sA + r2 * kAS + 32 + c2) = make_float4(a00.x, a00.y, a01.x, a01.y);
        *reinterpret_cast<float4 *>(sA + (r2 + 1) * kAS + 32 + c2) = make_float4(a10.x, a10.y, a11.x, a11.y);
    } else {
        for (int e = tid - 128; e < 32 * 16; e += kTh - 128) {
            const int r = e >> 4, c = (e & 15) * 4;
            float4 t4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c < 32) t4 = *reinterpret_cast<const float4 *>(sT + r * kAS + c);
            const float4 b4 = *reinterpret_cast<const float4 *>(s_beta + c);
            put_tb4_scaled(tb16, tbh, tbl, r, c, t4, b4);
        }
    }
    sync();
    // (2b) T[32 + r][0 .. 31] = -T_hi R, times beta, straight into Tb (T_hi is lower triangular: a
    //      warp's rows end at 8 warp + 7). Warps 4-15: Tb rows 32-63, columns 32-63 (T_hi times beta)
    if (warp < 4) {
        float2 a00 = make_float2(0.f, 0.f), a01 = a00, a10 = a00, a11 = a00;  // row, column pair
#pragma unroll 8
        for (int s = 0; s < 8 * warp + 8; ++s) {
            const float t0 = sT[(32 + r2) * kAS + 32 + s], t1 = sT[(33 + r2) * kAS + 32 + s];
            const float4 y = *reinterpret_cast<const float4 *>(sA + s * kAS + 32 + c2);
            const float2 ylo = make_float2(y.x, y.y), yhi = make_float2(y.z, y.w);
            a00 = fma2(make_float2(t0, t0), ylo, a00);
            a01 = fma2(make_float2(t0, t0), yhi, a01);
            a10 = fma2(make_float2(t1, t1), ylo, a10);
            a11 = fma2(make_float2(t1, t1), yhi, a11);
        }
        const float4 acc0 = make_float4(a00.x, a00.y, a01.x, a01.y), acc1 = make_float4(a10.x, a10.y, a11.x, a11.y);
        const float4 b4 = *reinterpret_cast<const float4 *>(s_beta + c2);
        put_tb4_scaled(tb16, tbh, tbl, 32 + r2, c2, make_float4(-acc0.x, -acc0.y, -acc0.z, -acc0.w), b4);
        put_tb4_scaled(tb16, tbh, tbl, 33 + r2, c2, make_float4(-acc1.x, -acc1.y, -acc1.z, -acc1.w), b4);
    } else {
        for (int e = tid - 128; e < 32 * 8; e += kTh - 128) {
            const int r = 32 + (e >> 3), c = 32 + (e & 7) * 4;
            const float4 t4 = *reinterpret_cast<const float4 *>(sT + r * kAS + c);
            const float4 b4 = *reinterpret_cast<const float4 *>(s_beta + c);
            put_tb4_scaled(tb16, tbh, tbl, r, c, t4, b4);
        }
    }
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// Bulk copy shared -> global by one thread, in the thread's current bulk group; both addresses
// 16-byte aligned, bytes a multiple of 16. The shared source must not change until
// bulk_wait_read has seen the group through.
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(reinterpret_cast<uint64_t>(dst)),
                 "r"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ------------------------------------------------------------------------------------------
// The prep: one CTA of 16 warps per SM walks the segment's (sequence, head, chunk) items, taken
// from a counter (CTAs that start late, behind other work on their SM, take fewer). Items are
// numbered chunk by chunk, (sequence, head) fastest, and item n's record is the n-th: the CTAs at
// work together read neighbouring heads of the same tokens, whole rows of q, k and alpha, instead
// of rows 16-32 KB apart (chunk-fastest numbering: 1.615 ms against 1.606 at 32K). Half the CTA
// forms an item's operands while the other half finishes the item before it, so the solve's long
// serial chain (run by four warps, the others waiting at its barriers) overlaps the next item's
// formation:
//   warps 0-7, the former: staging wait, decays and operand tiles ([Kt; Qt] into one of two
//     buffers, Kh), [Kt; Qt] Kh^T on the tensor cores, A (into one of two scratch buffers) and P;
//   warps 8-15, the solver: (I + A)^-1 and the Tb tiles, W = Tb Kt on the tensor cores, W out.
// An item passes from the former to the solver through buffer j % 2 (the [Kt; Qt] tile and the A
// scratch) with two mbarriers per buffer: full (the former's item is in it) and empty (the solver is
// done with it: its W MMA has read Kt, and the solve has read A). Each half synchronises on its own
// named barrier. The record leaves as each half finishes its part: the former's Qt and Kh (bulk,
// from their tiles), P (bulk, from a tile over the scan's buffer) and g_last; the solver's Tb hi /
// lo (stores from registers) and W (bulk, from a tile over the T scratch). Each half's bulk
// stores are its own, so neither waits on the other's. Every wait is bounded; the former ends the
// solver's loop with an item of -1.
// ------------------------------------------------------------------------------------------
constexpr uint32_t kWQW = 0;                          // [Kt; Qt] x 2, 32 KiB each (the record's Qt)
constexpr uint32_t kWKH = 65536;                      // Kh [64 tok][128 d_k], 2 blocks x 8 KiB
constexpr uint32_t kWSuf = 81920;                     // the decay scan's backward products [16][128] fp32
constexpr uint32_t kWSQ = 90112, kWSK = 106496, kWSA = 122880;  // q, k, alpha staging (TMA, plain)
constexpr uint32_t kWAStride = 64 * kAS * 4;          // one A / T scratch [64][kAS] fp32
constexpr uint32_t kWA = 155648;                      // A scratch x 2
constexpr uint32_t kWT = kWA + 2 * kWAStride;         // T scratch (the solver's)
constexpr uint32_t kWTB = kWT + kWAStride;            // Tb [64 r][64 s] fp16 K-major (the W MMA's A)
constexpr uint32_t kWMisc = kWTB + 8192;
constexpr uint32_t kWmBeta = 0, kWmBetaS = 256, kWmRq = 768, kWmRk = 1024, kWmRg = 1280, kWmOct = 1792,
                   kWmBar = kWmOct + 16 * 128 * 4, kWmTmem = kWmBar + 64, kWmAbort = kWmTmem + 4,
                   kWmFetch = kWmTmem + 8, kWmItem = kWmTmem + 16, kWmEnd = kWmTmem + 32;
constexpr uint32_t kWSmemBytes = kWMisc + kWmEnd + 1024;
static_assert(kWSmemBytes <= 232448, "prep shared memory over the per-block limit");
static_assert(kWTB % 1024 == 0 && kWQW % 1024 == 0 && kWKH % 1024 == 0, "swizzled tiles need 1024-byte alignment");
constexpr int kWHalf = 256;                           // threads of each half
constexpr int kWFetchTid = 128, kWStageTid = 32, kWBulkTid = 64;  // former threads with a side job
constexpr int kWSBulkTid = 32;  // the solver's thread (in its own numbering) that stores W in bulk
// TMEM columns: [Kt; Qt] Kh^T (the former's), W (the solver's)
constexpr uint32_t kWColA = 0, kWColW = 64, kWTmemCols = 256;

__device__ __forceinline__ void half_bar(int id) { asm volatile("bar.sync %0, 256;" ::"r"(id) : "memory"); }
// the AND of `v` over a half's 256 threads, at its named barrier
__device__ __forceinline__ bool half_and(int id, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "r"(id)
        : "memory");
    return r != 0;
}

template <bool kL2>  // kL2: q and k are L2-normalised per token (p.l2norm)
__global__ void __launch_bounds__(kPThreads, 1) kda_chunk_prep_ws_kernel(PrepArgs p,
                                                                         const __grid_constant__ PrepMaps maps) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint8_t *misc = sm + kWMisc;
    const uint32_t stage_bar = sbase + kWMisc + kWmBar, mmaf_bar = stage_bar + 8, mmas_bar = stage_bar + 16;
    const uint32_t full_bar = stage_bar + 24, empty_bar = stage_bar + 40;  // two each, 8 bytes apart
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + kWmTmem);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + kWmAbort);
    int *s_fetch = reinterpret_cast<int *>(misc + kWmFetch);
    volatile int *s_item = reinterpret_cast<volatile int *>(misc + kWmItem);  // per buffer: the item, or -1

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = warp & 3;  // TMEM sub-partition
    const uint32_t lane_base = static_cast<uint32_t>(32 * sp) << 16;
    const int nitems = p.B * p.H * p.nseg;
    const uint64_t d0 = smem_desc(sbase, 16, 1024, kLayoutSw128);

    if (tid == 0) {
        mbar_init(stage_bar, 1);
        mbar_init(mmaf_bar, 1);
        mbar_init(mmas_bar, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(full_bar + 8 * b, 1);
            mbar_init(empty_bar + 8 * b, 1);
        }
        *abort_flag = 0;
        s_fetch[0] = atomicAdd(p.counter, 1);  // the first item, and the one after it
        s_fetch[1] = atomicAdd(p.counter, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kWTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 8) {
        // ============================== the former ==============================
        const int ft = tid;  // 0-255
        float *s_beta = reinterpret_cast<float *>(misc + kWmBeta);
        float *s_rq = reinterpret_cast<float *>(misc + kWmRq);
        float *s_rk = reinterpret_cast<float *>(misc + kWmRk);
        float *s_rg = reinterpret_cast<float *>(misc + kWmRg);
        float *s_oct = reinterpret_cast<float *>(misc + kWmOct);
        float *s_suf = reinterpret_cast<float *>(sm + kWSuf);
        uint32_t stage_phase = 0, mma_phase = 0;
        bool ok = true;
        auto coords = [&](int item, int &b, int &h, int &ch) {
            const int bhn = p.B * p.H;
            const int cc = item / bhn;
            const int bh = item - cc * bhn;
            ch = p.c0 + cc;
            b = bh / p.H;
            h = bh - b * p.H;
        };
        auto stage_qka = [&](int b, int h, int ch) {
            fence_async_smem();
            mbar_arrive_tx_raw(stage_bar, kPStageTx);
            tma_load_3d(sbase + kWSQ, &maps.q, h * kDk, ch * kC, b, stage_bar);
            tma_load_3d(sbase + kWSK, &maps.k, h * kDk, ch * kC, b, stage_bar);
            tma_load_3d(sbase + kWSA, &maps.alpha, h * kDk, ch * kC, b, stage_bar);
        };
        auto load_beta = [&](int it, int b, int h, int ch) -> float {
            if (ft >= kC || it >= nitems) return 0.f;
            const int t = ch * kC + ft;
            return t < p.T ? p.beta[(static_cast<size_t>(b) * p.T + t) * p.H + h] : 0.f;
        };
        int item = s_fetch[0], next = s_fetch[1];
        int nb, nh, nch;
        coords(item, nb, nh, nch);
        float beta_next = load_beta(item, nb, nh, nch);
        int pending = 0;
        if (item < nitems) {
            if (ft == kWStageTid) stage_qka(nb, nh, nch);
            pending = 1;
        }
        for (int j = 0;; ++j) {
            const int bf = j & 1;
            // the buffer's previous item (j - 2) must be done with: the solver's W has read its Kt and
            // its solve its A
            if (j >= 2) {
                bool w = true;
                if (warp == 0)
                    w = wait_bar(empty_bar + 8 * bf, static_cast<uint32_t>((j - 2) >> 1) & 1u, abort_flag,
                                 &g_prefill_error, lad::kErrPrefill);
                ok = half_and(1, w && ok);
            }
            if (item >= nitems || !ok) {
                if (ft == 0) {
                    s_item[bf] = -1;
                    mbar_arrive(full_bar + 8 * bf);
                }
                break;
            }
            const int ch = nch;
            coords(next, nb, nh, nch);
            // the next item's q, k and alpha start for L2 now; they are staged (TMA) only once this
            // item's formation has read the staging buffers
            if (ft == kWStageTid && next < nitems) {
                tma_prefetch_3d(&maps.q, nh * kDk, nch * kC, nb);
                tma_prefetch_3d(&maps.k, nh * kDk, nch * kC, nb);
                tma_prefetch_3d(&maps.alpha, nh * kDk, nch * kC, nb);
            }
            const int t0 = ch * kC;
            const int n = min(kC, p.T - t0);
            uint8_t *rec = p.ws + static_cast<size_t>(item) * kRecBytes;
            float *sA = reinterpret_cast<float *>(sm + kWA + bf * kWAStride);
            float *s_betaS = reinterpret_cast<float *>(misc + kWmBetaS) + bf * kC;
            const uint32_t qw = kWQW + bf * 32768u;

            if (ft < kC) {
                s_beta[ft] = beta_next;
                s_betaS[ft] = beta_next;
            }
            beta_next = load_beta(next, nb, nh, nch);
            {
                bool w = true;
                if (warp == 0) w = wait_bar(stage_bar, stage_phase, abort_flag, &g_prefill_error, lad::kErrPrefill);
                stage_phase ^= 1;
                pending = 0;
                ok = half_and(1, w);
                if (!ok) {
                    if (ft == 0) {
                        s_item[bf] = -1;
                        mbar_arrive(full_bar + 8 * bf);
                    }
                    break;
                }
            }
            const uint16_t *sq = reinterpret_cast<const uint16_t *>(sm + kWSQ);
            const uint16_t *sk = reinterpret_cast<const uint16_t *>(sm + kWSK);
            const float *sa = reinterpret_cast<const float *>(sm + kWSA);
            if constexpr (kL2) {
#pragma unroll 1
                for (int r = warp; r < kC; r += 8) {
                    const uint2 qv = *reinterpret_cast<const uint2 *>(sq + r * kDk + 4 * lane);
                    const uint2 kv = *reinterpret_cast<const uint2 *>(sk + r * kDk + 4 * lane);
                    const float2 q0 = lad::dev::bf16x2_to_f32(qv.x), q1 = lad::dev::bf16x2_to_f32(qv.y);
                    const float2 k0 = lad::dev::bf16x2_to_f32(kv.x), k1 = lad::dev::bf16x2_to_f32(kv.y);
                    float sqs = q0.x * q0.x + q0.y * q0.y + q1.x * q1.x + q1.y * q1.y;
                    float sks = k0.x * k0.x + k0.y * k0.y + k1.x * k1.x + k1.y * k1.y;
#pragma unroll
                    for (int o = 16; o; o >>= 1) {
                        sqs += __shfl_xor_sync(0xffffffffu, sqs, o);
                        sks += __shfl_xor_sync(0xffffffffu, sks, o);
                    }
                    if (lane == 0) {
                        s_rq[r] = rsqrtf(sqs + 1e-6f);
                        s_rk[r] = rsqrtf(sks + 1e-6f);
                    }
                }
            }
            // ---- the decays and the operand tiles. Per key channel, g_r = prod_{s <= r} alpha_s and
            //      R_r = prod_{s > r} alpha_s, so that Kh = K R / g_last takes one reciprocal per channel
            //      and none per element. Warp w takes the two quartets 2w, 2w + 1 (tokens 8w .. 8w+7),
            //      lane l the channels 4l .. 4l+3: the quartets' products first; threads 0-127 scan a
            //      channel's 16 quartet products both ways; then each quartet's running products again
            //      (from alpha) and its four tokens ----
            const int c4 = 4 * lane;
            auto quartet_products = [&](int o, float4 (&fw)[4], float4 (&bw)[4]) {
                float4 a4[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int r = 4 * o + u;
                    a4[u] = (r < n) ? *reinterpret_cast<const float4 *>(sa + r * kDk + c4) : make_float4(1.f, 1.f, 1.f, 1.f);
                }
                float2 r01 = make_float2(1.f, 1.f), r23 = r01;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    r01 = mul2(r01, make_float2(a4[u].x, a4[u].y));
                    r23 = mul2(r23, make_float2(a4[u].z, a4[u].w));
                    fw[u] = make_float4(r01.x, r01.y, r23.x, r23.y);
                }
                r01 = r23 = make_float2(1.f, 1.f);
#pragma unroll
                for (int u = 3; u >= 0; --u) {
                    bw[u] = make_float4(r01.x, r01.y, r23.x, r23.y);
                    r01 = mul2(r01, make_float2(a4[u].x, a4[u].y));
                    r23 = mul2(r23, make_float2(a4[u].z, a4[u].w));
                }
            };
#pragma unroll 1
            for (int qq = 0; qq < 2; ++qq) {
                float4 fw[4], bw[4];
                quartet_products(2 * warp + qq, fw, bw);
                *reinterpret_cast<float4 *>(s_oct + (2 * warp + qq) * kDk + c4) = fw[3];
            }
            // the previous item's bulk stores have read Qt, Kh and P (their regions are written next)
            if (ft == kWBulkTid) bulk_wait_read0();
            half_bar(1);
            if (ft < kDk) {
                float y[16];
#pragma unroll
                for (int oo = 0; oo < 16; ++oo) y[oo] = s_oct[oo * kDk + ft];
                float pre = 1.f, suf = 1.f;
#pragma unroll
                for (int oo = 0; oo < 16; ++oo) {
                    s_oct[oo * kDk + ft] = pre;  // before quartet oo
                    pre *= y[oo];
                    s_suf[(15 - oo) * kDk + ft] = suf;  // after quartet 15 - oo
                    suf *= y[15 - oo];
                }
                reinterpret_cast<float *>(rec + kRG)[ft] = pre;  // g_last, for the record
                s_rg[ft] = __frcp_rn(pre);
            }
            half_bar(1);
            const float4 rg = *reinterpret_cast<const float4 *>(s_rg + c4);
            const float2 rg01 = make_float2(rg.x, rg.y), rg23 = make_float2(rg.z, rg.w);
#pragma unroll 1
            for (int qq = 0; qq < 2; ++qq) {
                const int o = 2 * warp + qq;
                float4 fw[4], bw[4];
                quartet_products(o, fw, bw);
                const float4 ex = *reinterpret_cast<const float4 *>(s_oct + o * kDk + c4);
                const float4 sx = *reinterpret_cast<const float4 *>(s_suf + o * kDk + c4);
                const float2 ex01 = make_float2(ex.x, ex.y), ex23 = make_float2(ex.z, ex.w);
                const float2 sx01 = make_float2(sx.x, sx.y), sx23 = make_float2(sx.z, sx.w);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int r = 4 * o + u;
                    const float2 g01 = mul2(ex01, make_float2(fw[u].x, fw[u].y));
                    const float2 g23 = mul2(ex23, make_float2(fw[u].z, fw[u].w));
                    const float2 R01 = mul2(sx01, make_float2(bw[u].x, bw[u].y));
                    const float2 R23 = mul2(sx23, make_float2(bw[u].z, bw[u].w));
                    const uint2 qv = *reinterpret_cast<const uint2 *>(sq + r * kDk + c4);
                    const uint2 kv = *reinterpret_cast<const uint2 *>(sk + r * kDk + c4);
                    float2 q01 = lad::dev::bf16x2_to_f32(qv.x), q23 = lad::dev::bf16x2_to_f32(qv.y);
                    float2 k01 = lad::dev::bf16x2_to_f32(kv.x), k23 = lad::dev::bf16x2_to_f32(kv.y);
                    if constexpr (kL2) {
                        const float rq = s_rq[r], rk = s_rk[r];
                        q01 = mul2(q01, make_float2(rq, rq));
                        q23 = mul2(q23, make_float2(rq, rq));
                        k01 = mul2(k01, make_float2(rk, rk));
                        k23 = mul2(k23, make_float2(rk, rk));
                    }
                    const float2 kh01 = mul2(mul2(k01, R01), rg01), kh23 = mul2(mul2(k23, R23), rg23);
                    const float2 kt01 = mul2(k01, g01), kt23 = mul2(k23, g23);
                    const float2 qt01 = mul2(q01, g01), qt23 = mul2(q23, g23);
                    const uint32_t off = sw128_off16(r, c4, 8192);         // Kh, a 64-row tile
                    const uint32_t offq = sw128_off16(kC + r, c4, 16384);  // row 64 + r of [Kt; Qt]
                    const uint32_t offk = sw128_off16(r, c4, 16384);       // row r of [Kt; Qt]
                    *reinterpret_cast<uint2 *>(sm + qw + offk) =
                        make_uint2(f32x2_to_f16x2(kt01.x, kt01.y), f32x2_to_f16x2(kt23.x, kt23.y));
                    *reinterpret_cast<uint2 *>(sm + qw + offq) =
                        make_uint2(f32x2_to_f16x2(qt01.x, qt01.y), f32x2_to_f16x2(qt23.x, qt23.y));
                    *reinterpret_cast<uint2 *>(sm + kWKH + off) =
                        make_uint2(f32x2_to_f16x2(kh01.x, kh01.y), f32x2_to_f16x2(kh23.x, kh23.y));
                }
            }
            // ---- [Kt; Qt] Kh^T: rows 0-63 give Kt Kh^T, rows 64-127 Qt Kh^T ----
            fence_async_smem();
            tc_fence_before();
            half_bar(1);  // q, k and alpha of this item are read: the next item's come in
            if (next < nitems) {
                if (ft == kWStageTid) stage_qka(nb, nh, nch);
                pending = 1;
            }
            if (ft == kWFetchTid) s_fetch[0] = atomicAdd(p.counter, 1);  // read after this item's last barrier
            if (ft == kWBulkTid) {  // the record's Qt (rows 64-127 of each block of the tile) and Kh
                bulk_s2g(rec + kRWQ + 8192, sbase + qw + 8192, 8192);
                bulk_s2g(rec + kRWQ + 16384 + 8192, sbase + qw + 16384 + 8192, 8192);
                bulk_s2g(rec + kRKH, sbase + kWKH, 16384);
                bulk_commit();
            }
            if (warp == 0) {
                tc_fence_after();
#pragma unroll
                for (int jj = 0; jj < kDk / 16; ++jj)
                    tc_mma_f16(tmem + kWColA, kdesc16(d0 + (qw >> 4), 16384, jj), kdesc16(d0 + (kWKH >> 4), 8192, jj),
                               kIdescA, jj > 0);
                tc_commit(mmaf_bar);
            }
            {
                bool w = true;
                if (warp == 0) w = wait_bar(mmaf_bar, mma_phase, abort_flag, &g_prefill_error, lad::kErrPrefill);
                mma_phase ^= 1;
                ok = half_and(1, w);
                tc_fence_after();
                if (!ok) {
                    if (ft == 0) {
                        s_item[bf] = -1;
                        mbar_arrive(full_bar + 8 * bf);
                    }
                    break;
                }
            }
            // ---- A = strict_lower(diag(beta) Kt Kh^T) -> fp32 scratch; P = lower(Qt Kh^T) -> fp16 tile
            //      over the scan's buffer (read by now), stored to the record in bulk; a warp takes 32 of
            //      a row's 64 columns, in two 16-column loads ----
#pragma unroll 1
            for (int qq = 0; qq < 2; ++qq) {
                const int qd = 2 * (warp >> 2) + qq;
                float x[16];
                tmem_ld16(tmem + lane_base + kWColA + 16 * qd, x);
                tmem_wait_ld();
                const int row = 32 * sp + lane, c0 = 16 * qd;
                if (row < kC) {
                    const int r = row;
                    const float br = s_beta[r];
                    float4 *dst = reinterpret_cast<float4 *>(sA + r * kAS + c0);
#pragma unroll
                    for (int jj = 0; jj < 16; jj += 4) {
                        const float2 p01 = mul2(make_float2(br, br), make_float2(x[jj], x[jj + 1]));
                        const float2 p23 = mul2(make_float2(br, br), make_float2(x[jj + 2], x[jj + 3]));
                        dst[jj / 4] = make_float4(c0 + jj < r ? p01.x : 0.f, c0 + jj + 1 < r ? p01.y : 0.f,
                                                  c0 + jj + 2 < r ? p23.x : 0.f, c0 + jj + 3 < r ? p23.y : 0.f);
                    }
                } else {
                    const int r = row - kC;
#pragma unroll
                    for (int jj = 0; jj < 16; jj += 8) {
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = (c0 + jj + e <= r) ? x[jj + e] : 0.f;
                        *reinterpret_cast<uint4 *>(sm + kWSuf + sw128_off16(r, c0 + jj, 8192)) =
                            make_uint4(f32x2_to_f16x2(y[0], y[1]), f32x2_to_f16x2(y[2], y[3]),
                                       f32x2_to_f16x2(y[4], y[5]), f32x2_to_f16x2(y[6], y[7]));
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            half_bar(1);  // A and beta of the item are in place (and TMEM's column block is read)
            if (ft == 0) {
                s_item[bf] = item;
                mbar_arrive(full_bar + 8 * bf);
            }
            if (ft == kWBulkTid) {
                bulk_s2g(rec + kRP, sbase + kWSuf, 8192);
                bulk_commit();
            }
            item = next;
            next = s_fetch[0];
        }
        // drain: a staging copy still in flight (after an abort) lands and the bulk stores complete
        if (ft == 0 && pending) {
            const uint64_t t0 = lad::dev::globaltimer_ns();
            while (!mbar_try_wait(stage_bar, stage_phase) && lad::dev::globaltimer_ns() - t0 < lad::dev::kWaitLimitNs) {
            }
        }
        if (ft == kWBulkTid) bulk_wait_all();
        // every [Kt; Qt] Kh^T MMA has completed (after an abort, a fresh commit is waited for, bounded)
        if (warp == 0) {
            tc_commit(mmaf_bar);
            if (lane == 0) {
                const uint64_t t0 = lad::dev::globaltimer_ns();
                while (!mbar_try_wait(mmaf_bar, mma_phase) && lad::dev::globaltimer_ns() - t0 < lad::dev::kWaitLimitNs) {
                }
            }
            __syncwarp();
        }
    } else {
        // ============================== the solver ==============================
        const int st = tid - kWHalf;  // 0-255
        const int sw = st >> 5;       // the solver's warp, 0-7
        float *sT = reinterpret_cast<float *>(sm + kWT);
        uint32_t mma_phase = 0;
        for (int j = 0;; ++j) {
            const int bf = j & 1;
            bool w = true;
            if (sw == 0)
                w = wait_bar(full_bar + 8 * bf, static_cast<uint32_t>(j >> 1) & 1u, abort_flag, &g_prefill_error,
                             lad::kErrPrefill);
            if (st == kWSBulkTid) bulk_wait_read0();  // the previous W has left the T scratch
            if (!half_and(2, w)) break;
            const int item = s_item[bf];
            if (item < 0) break;
            uint8_t *rec = p.ws + static_cast<size_t>(item) * kRecBytes;
            float *sA = reinterpret_cast<float *>(sm + kWA + bf * kWAStride);
            const float *s_betaS = reinterpret_cast<const float *>(misc + kWmBetaS) + bf * kC;
            // ---- T = (I + A)^-1, Tb = T diag(beta): the fp16 tile here, the bf16 hi / lo pair straight
            //      into the record ----
            solve_tb<kWHalf>(sA, sT, s_betaS, sm + kWTB, rec + kRTH, rec + kRTL, st, []() { half_bar(2); });
            // ---- W = Tb Kt (Kt: rows 0-63 of the buffer's [Kt; Qt], read MN-major) ----
            fence_async_smem();
            tc_fence_before();
            half_bar(2);
            if (sw == 0) {
                tc_fence_after();
                const uint64_t kt0 = smem_desc(sbase + kWQW + bf * 32768u, 16384, 1024, kLayoutSw128);
#pragma unroll
                for (int jj = 0; jj < kC / 16; ++jj)
                    tc_mma_f16(tmem + kWColW, kdesc16(d0 + (kWTB >> 4), 8192, jj), kt0 + ((jj * 2048) >> 4), kIdescW,
                               jj > 0);
                tc_commit(mmas_bar);
            }
            bool w2 = true;
            if (sw == 0) w2 = wait_bar(mmas_bar, mma_phase, abort_flag, &g_prefill_error, lad::kErrPrefill);
            mma_phase ^= 1;
            const bool ok = half_and(2, w2);
            tc_fence_after();
            if (!ok) break;
            if (st == 0) mbar_arrive(empty_bar + 8 * bf);  // the buffer's Kt and A are free
            // ---- W -> fp16 tile over the T scratch (the solve is done with it), then the record's
            //      [W; Qt] tile (rows 0-63 of each block) in bulk. M = 64: row 16 sp + i sits in lane i
            //      (< 16) of sub-partition sp; the loads are collective, so the whole warp issues them
            //      and lanes 0-15 keep the rows. A warp takes 64 of the 128 columns ----
#pragma unroll 1
            for (int qq = 0; qq < 2; ++qq) {
                const int c0 = 64 * (sw >> 2) + 32 * qq;
                float wv[32];
                tmem_ld32(tmem + lane_base + kWColW + c0, wv);
                tmem_wait_ld();
                if (lane < 16) {
                    const int r = 16 * sp + lane;
#pragma unroll
                    for (int jj = 0; jj < 32; jj += 8)
                        *reinterpret_cast<uint4 *>(sm + kWT + sw128_off16(r, c0 + jj, 8192)) =
                            make_uint4(f32x2_to_f16x2(wv[jj], wv[jj + 1]), f32x2_to_f16x2(wv[jj + 2], wv[jj + 3]),
                                       f32x2_to_f16x2(wv[jj + 4], wv[jj + 5]), f32x2_to_f16x2(wv[jj + 6], wv[jj + 7]));
                }
            }
            fence_async_smem();
            tc_fence_before();  // the W loads are done before the next item's W MMA
            half_bar(2);
            if (st == kWSBulkTid) {
                bulk_s2g(rec + kRWQ, sbase + kWT, 8192);
                bulk_s2g(rec + kRWQ + 16384, sbase + kWT + 8192, 8192);
                bulk_commit();
            }
        }
        if (st == kWSBulkTid) bulk_wait_all();
        // every W MMA has completed (after an abort, a fresh commit is waited for, bounded)
        if (sw == 0) {
            tc_commit(mmas_bar);
            if (lane == 0) {
                const uint64_t t0 = lad::dev::globaltimer_ns();
                while (!mbar_try_wait(mmas_bar, mma_phase) && lad::dev::globaltimer_ns() - t0 < lad::dev::kWaitLimitNs) {
                }
            }
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kWTmemCols);
}

struct ChainArgs {
    float *S;
    void *o;
    const uint8_t *ws;  // this segment's records, [B*H][nseg]
    int B, T, H;
    int c0, nseg;
    float scale;
    int out_f32;
};

// chain shared memory (offsets from a 1024-aligned base)
constexpr uint32_t kCS16 = 0;            // S0^T [128 d_v][128 d_k] fp16, K-major SW128, 2 blocks x 16 KiB
constexpr uint32_t kCRec = 32768;        // two chunk buffers: the record, then the chunk's v tile
constexpr uint32_t kCV = 74752;          // in a buffer: v [64 tok][128 d_v] bf16 (TMA, SW128, two blocks
                                         //   of 64 d_v: the MN-major operand), then U^T [128 d_v][64 tok] fp16
constexpr uint32_t kCRecStride = kCV + 16384;  // 89 KiB (1024-aligned); the barriers sit in buffer 0's slack
constexpr uint32_t kCO = kCRec + 2 * kCRecStride;  // O [64 tok][128 d_v] bf16 (or 32 tokens x fp32), plain
constexpr uint32_t kCMisc = kCRec + kRecBytes;     // buffer 0's 512 bytes between record and v tile: 2 chunk
                                                   // barriers, 3 MMA barriers, TMEM slot, abort
constexpr uint32_t kCSmemBytes = kCO + 16384 + 1024;
static_assert(kCMisc + 64 <= kCRec + kCV, "chain barriers must fit in the record slack");
static_assert(kRecBytes + 512 <= kCV, "the g_last copy must fit in buffer 1's slack");
static_assert(kCV % 1024 == 0 && kCRecStride % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(kCSmemBytes <= 232448, "chain shared memory over the per-block limit");
constexpr uint32_t kCChunkTx = kRecBytes + 16384;  // a chunk buffer's bytes: the record and the v tile
constexpr uint32_t kCGl = kCRec + kCRecStride + kRecBytes;  // buffer 1's slack: the current chunk's g_last,
                                                            // copied out before its buffer is refilled
// TMEM: the fp32 master S^T (128 lanes = d_v, 128 columns = d_k), two [X^T | O^T] buffers of
// 128 columns (chunk parity), U'^T (64 columns)
constexpr uint32_t kCColS = 0, kCColXO = 128, kCColU = 384, kCTmemCols = 512;

struct ChainMaps {
    CUtensorMap o;  // o as [B][T][H * 128] (bf16, or fp32), boxes of 128 channels x 64 (32) tokens
    CUtensorMap v;  // v as [B][T][H * 128] bf16, boxes of 64 channels x 64 tokens, 128-byte swizzle
};

__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, uint32_t src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// One CTA per (sequence, head) walks the segment's chunks with the state master in tensor memory.
// Warps 0-7 own the master's rows (warp w: lanes 32 (w % 4) .., columns half w / 4); warp 8 issues
// the MMAs and the chunk copies (the record by one bulk copy, the v tile by two TMA loads, two
// chunks ahead). Per chunk: the first batch ([X^T | O^T] from S0's fp16 copy, U'^T; one commit),
// while warps 0-7 send the previous chunk's outputs out; warps 0-7 form U^T = U'^T - X^T as the
// fp16 operand over the v tile and meet warp 8 at a named barrier; the second batch (the state
// part, its own commit, then the rest of O^T, a third); warps 0-7 then read the new master, write
// its fp16 copy over S0's (the first batch, its only reader, is complete) and scale the master by
// the next chunk's decay. The threads touch tensor memory while the tensor cores are idle where
// they can: a decay pass run beside the first batch took three times as long.
constexpr int kChainThreads = kThreads + 32;

__global__ void __launch_bounds__(kChainThreads, 1) kda_chunk_chain_kernel(ChainArgs p,
                                                                          const __grid_constant__ ChainMaps maps) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    // mbar_a: the first batch; mbar_s: the state part of the second; mbar_p: every MMA of the chunk
    const uint32_t rec_bar0 = sbase + kCMisc, mbar_s = sbase + kCMisc + 16, mbar_a = sbase + kCMisc + 24,
                   mbar_p = sbase + kCMisc + 40;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kCMisc + 32);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kCMisc + 36);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool issuer = warp == kThreads / 32;  // warp 8
    const int sp = warp & 3, cg = (warp >> 2) & 1;
    const uint32_t lane_base = static_cast<uint32_t>(32 * sp) << 16;
    const int dv = 32 * sp + lane;  // this thread's row of S^T: a value column (warps 0-7)
    const int bh = blockIdx.x;
    const int b = bh / p.H, h = bh - b * p.H;
    const uint8_t *recs = p.ws + static_cast<size_t>(bh) * kRecBytes;
    const size_t rec_stride = static_cast<size_t>(p.B) * p.H * kRecBytes;  // chunk i's record: recs + i * this
    const uint64_t d0 = smem_desc(sbase, 16, 1024, kLayoutSw128);

    if (tid == 0) {
        mbar_init(rec_bar0, 1);
        mbar_init(rec_bar0 + 8, 1);
        mbar_init(mbar_s, 1);
        mbar_init(mbar_a, 1);
        mbar_init(mbar_p, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kCTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // chunk i's record and v tile into buffer i % 2 (one thread); the v rows past T read as zero
    auto load_chunk = [&](int i) {
        const uint32_t bar = rec_bar0 + 8u * static_cast<uint32_t>(i & 1);
        const uint32_t buf = sbase + kCRec + static_cast<uint32_t>(i & 1) * kCRecStride;
        mbar_arrive_tx_raw(bar, kCChunkTx);
        bulk_g2s(buf, recs + static_cast<size_t>(i) * rec_stride, kRecBytes, bar);
        const int t0 = (p.c0 + i) * kC;
        tma_load_3d(buf + kCV, &maps.v, h * kDv, t0, b, bar);
        tma_load_3d(buf + kCV + 8192, &maps.v, h * kDv + 64, t0, b, bar);
    };
    uint32_t pend = p.nseg > 1 ? 3u : 1u;  // bit j: a copy into buffer j is in flight (issuer's view)
    if (issuer && lane == 0) {
        load_chunk(0);
        if (p.nseg > 1) load_chunk(1);
    }
    // waits by the calling warp (bounded; warp-uniform result); chunk i's buffer has landed
    auto rec_ready = [&](int i) {
        const int j = i & 1;
        return wait_bar(rec_bar0 + 8u * j, static_cast<uint32_t>(i >> 1) & 1u, abort_flag, &g_prefill_error,
                        lad::kErrPrefill);
    };
    auto gl_of = [&](int i) {  // g_last of chunk i (its record buffer)
        return reinterpret_cast<const float *>(sm + kCRec + static_cast<uint32_t>(i & 1) * kCRecStride + kRG);
    };
    auto bar256 = []() { asm volatile("bar.sync 1, 256;" ::: "memory"); };  // warps 0-7 only
    auto bar288 = []() { asm volatile("bar.sync 2, 288;" ::: "memory"); };  // warps 0-8
    // O of chunk i (O^T in buffer i % 2, complete), scaled, through the O tile and TMA stores;
    // warps 0-7, the previous store having read the tile
    auto store_o = [&](int i) {
        float x[32];
        tmem_ld32(tmem + lane_base + kCColXO + static_cast<uint32_t>(i & 1) * 128 + 64 + 32 * cg, x);
        tmem_wait_ld();
        const int t0 = (p.c0 + i) * kC;
        if (!p.out_f32) {
            // a lane pair (d_v, d_v + 1) trades values so that each lane writes a bf16 pair of one
            // token: the even lane token j, the odd lane token j + 1 (one packed conversion and one
            // 4-byte store per two values)
            const int odd = lane & 1;
            uint32_t *od = reinterpret_cast<uint32_t *>(sm + kCO) + ((32 * cg + odd) * kDv + dv - odd) / 2;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                const float2 mine = mul2(make_float2(p.scale, p.scale), make_float2(x[j], x[j + 1]));
                const float other = __shfl_xor_sync(0xffffffffu, odd ? mine.x : mine.y, 1);
                od[j * (kDv / 2)] = odd ? bf16x2_rn(other, mine.y) : bf16x2_rn(mine.x, other);
            }
            fence_async_smem();
            bar256();
            if (tid == 0) {
                tma_store_3d(&maps.o, sbase + kCO, h * kDv, t0, b);
                bulk_commit();
            }
        } else {
            // fp32: 32 tokens (16 KiB) at a time, the two column halves one after the other
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                if (cg == half) {
                    float *od = reinterpret_cast<float *>(sm + kCO) + dv;
#pragma unroll
                    for (int j = 0; j < 32; ++j) od[j * kDv] = p.scale * x[j];
                    fence_async_smem();
                }
                bar256();
                if (tid == 0) {
                    tma_store_3d(&maps.o, sbase + kCO, h * kDv, t0 + 32 * half, b);
                    bulk_commit();
                    bulk_wait_read0();
                }
                bar256();
            }
        }
    };

    // ---- the state entering the segment: the fp16 copy (S0^T) and the fp32 master ----
    bool ok = true;
    if (!issuer) {
        ok = rec_ready(0);
        if (ok) {
            const float *S0 = p.S + static_cast<size_t>(bh) * kDk * kDv + dv;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const int c0 = 64 * cg + 32 * part;
                float v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = S0[static_cast<size_t>(c0 + j) * kDv];
#pragma unroll
                for (int j = 0; j < 32; j += 8)
                    *reinterpret_cast<uint4 *>(sm + kCS16 + sw128_off16(dv, c0 + j, 16384)) =
                        make_uint4(f32x2_to_f16x2(v[j], v[j + 1]), f32x2_to_f16x2(v[j + 2], v[j + 3]),
                                   f32x2_to_f16x2(v[j + 4], v[j + 5]), f32x2_to_f16x2(v[j + 6], v[j + 7]));
                tmem_st32(tmem + lane_base + kCColS + c0, v);
            }
            tmem_wait_st();
        }
    }
    fence_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok) != 0;
    tc_fence_after();


    for (int i = 0; i < p.nseg && ok; ++i) {
        const uint32_t rs = kCRec + static_cast<uint32_t>(i & 1) * kCRecStride;  // this chunk's buffer
        const uint32_t xo = tmem + kCColXO + static_cast<uint32_t>(i & 1) * 128;  // [X^T | O^T]
        const bool last = i == p.nseg - 1;
        bool w = true;
        if (issuer) {
            // ---- first batch: [X^T | O^T] = S0^T [W; Qt]^T, U'^T = V^T (Tb_hi + Tb_lo)^T ----
            tc_fence_after();
            const uint64_t sa0 = d0 + (kCS16 >> 4);
            const uint64_t v0 = smem_desc(sbase + rs + kCV, 8192, 1024, kLayoutSw128);  // MN chunks 8 KiB apart
#pragma unroll
            for (int j = 0; j < kDk / 16; ++j)
                tc_mma_f16(xo, kdesc16(sa0, 16384, j), kdesc16(d0 + ((rs + kRWQ) >> 4), 16384, j), kIdescXO, j > 0);
#pragma unroll
            for (int j = 0; j < kC / 16; ++j)
                tc_mma_f16(tmem + kCColU, v0 + ((j * 2048) >> 4), kdesc16(d0 + ((rs + kRTH) >> 4), 8192, j), kIdescU,
                           j > 0);
#pragma unroll
            for (int j = 0; j < kC / 16; ++j)
                tc_mma_f16(tmem + kCColU, v0 + ((j * 2048) >> 4), kdesc16(d0 + ((rs + kRTL) >> 4), 8192, j), kIdescU,
                           1);
            tc_commit(mbar_a);
            bar288();  // U^T is in place (over the v tile)
            tc_fence_after();
            // ---- second batch: S^T += U^T Kh (commit: the master pass may start); O^T += U^T P^T
            //      (commit: waited for here) ----
            const uint64_t ut0 = d0 + ((rs + kCV) >> 4);
            const uint64_t kg0 = smem_desc(sbase + rs + kRKH, 8192, 1024, kLayoutSw128);
#pragma unroll
            for (int j = 0; j < kC / 16; ++j)
                tc_mma_f16(tmem + kCColS, kdesc16(ut0, 16384, j), kg0 + ((j * 2048) >> 4), kIdescSU, 1);
            tc_commit(mbar_s);
#pragma unroll
            for (int j = 0; j < kC / 16; ++j)
                tc_mma_f16(xo + 64, kdesc16(ut0, 16384, j), kdesc16(d0 + ((rs + kRP) >> 4), 8192, j), kIdescO, 1);
            tc_commit(mbar_p);
            // every MMA of the chunk is complete: its buffer takes chunk i + 2's (and the barrier
            // below publishes the outputs, stored while the next chunk's first batch runs)
            w = wait_bar(mbar_p, static_cast<uint32_t>(i) & 1u, abort_flag, &g_prefill_error, lad::kErrPrefill);
            if (w && i + 2 < p.nseg) {
                if (lane == 0) load_chunk(i + 2);
                pend |= 1u << (i & 1);
            }
        } else {
            // ---- while the first batch runs: the previous chunk's outputs leave ----
            if (i > 0) store_o(i - 1);
            w = wait_bar(mbar_a, static_cast<uint32_t>(i) & 1u, abort_flag, &g_prefill_error, lad::kErrPrefill);
            tc_fence_after();
            // ---- U^T = U'^T - X^T -> the fp16 operand, over the v tile (its reader is complete). The
            //      chunk's g_last is copied out of its buffer too: the buffer takes chunk i + 2's
            //      record once this chunk's MMAs are complete, before the master pass reads it ----
            if (tid < kDk) reinterpret_cast<float *>(sm + kCGl)[tid] = gl_of(i)[tid];
            if (w) {
                float x[32], u[32];  // both loads before the one wait
                tmem_ld32(xo + lane_base + 32 * cg, x);
                tmem_ld32(tmem + lane_base + kCColU + 32 * cg, u);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 8)
                {
                    uint32_t h[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 d = sub2(make_float2(u[j + 2 * e], u[j + 2 * e + 1]),
                                              make_float2(x[j + 2 * e], x[j + 2 * e + 1]));
                        h[e] = f32x2_to_f16x2(d.x, d.y);
                    }
                    *reinterpret_cast<uint4 *>(sm + rs + kCV + sw128_off16(dv, 32 * cg + j, 16384)) =
                        make_uint4(h[0], h[1], h[2], h[3]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            bar288();
            if (w) w = wait_bar(mbar_s, static_cast<uint32_t>(i) & 1u, abort_flag, &g_prefill_error, lad::kErrPrefill);
            if (w && !last) w = rec_ready(i + 1);  // the next chunk's operands
            tc_fence_after();
            if (w) {
                // ---- the new state S = (S0 + Kh^T U) Diag(g_last): the chunk's decay on the master
                //      in fp32, then its fp16 copy over S0's (the first batch, S0's only reader, is
                //      complete), or the state out; both halves of the thread's row are loaded before
                //      the one wait ----
                float vv[2][32];
                tmem_ld32(tmem + lane_base + kCColS + 64 * cg, vv[0]);
                tmem_ld32(tmem + lane_base + kCColS + 64 * cg + 32, vv[1]);
                tmem_wait_ld();
                const float4 *gn = reinterpret_cast<const float4 *>(sm + kCGl) + 16 * cg;
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const int c0 = 64 * cg + 32 * part;
                    float (&v)[32] = vv[part];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 g4 = gn[8 * part + j];
                        const float2 a = mul2(make_float2(v[4 * j], v[4 * j + 1]), make_float2(g4.x, g4.y));
                        const float2 c = mul2(make_float2(v[4 * j + 2], v[4 * j + 3]), make_float2(g4.z, g4.w));
                        v[4 * j] = a.x;
                        v[4 * j + 1] = a.y;
                        v[4 * j + 2] = c.x;
                        v[4 * j + 3] = c.y;
                    }
                    if (last) {
                        float *Sout = p.S + static_cast<size_t>(bh) * kDk * kDv + dv;
#pragma unroll
                        for (int j = 0; j < 32; ++j) Sout[static_cast<size_t>(c0 + j) * kDv] = v[j];
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; j += 8)
                            *reinterpret_cast<uint4 *>(sm + kCS16 + sw128_off16(dv, c0 + j, 16384)) =
                                make_uint4(f32x2_to_f16x2(v[j], v[j + 1]), f32x2_to_f16x2(v[j + 2], v[j + 3]),
                                           f32x2_to_f16x2(v[j + 4], v[j + 5]), f32x2_to_f16x2(v[j + 6], v[j + 7]));
                        tmem_st32(tmem + lane_base + kCColS + c0, v);
                    }
                }
                tmem_wait_st();
            }
            if (tid == 0) bulk_wait_read0();  // the previous outputs have left the O tile
        }
        fence_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(w) != 0;
        tc_fence_after();
        if (ok && last && !issuer) store_o(i);
    }
    // drain: chunk copies still in flight (after an abort) land, the output stores complete and
    // every MMA this CTA issued completes, before shared memory and TMEM are released
    if (issuer) {
        if (lane == 0) {
            const uint64_t t0 = lad::dev::globaltimer_ns();
            for (int j = 0; j < 2; ++j) {
                // wait on the phase of the newest chunk that used buffer j
                const int newest = ((p.nseg - 1) & 1) == j ? p.nseg - 1 : p.nseg - 2;
                if (newest < 0) continue;
                while (((pend >> j) & 1u) &&
                       !mbar_try_wait(rec_bar0 + 8u * j, static_cast<uint32_t>(newest >> 1) & 1u) &&
                       lad::dev::globaltimer_ns() - t0 < lad::dev::kWaitLimitNs) {
                }
            }
        }
        __syncwarp();
        tc_commit(mbar_a);  // warp-wide (elect.sync): a fresh completion covering every MMA issued
        if (lane == 0) {
            const uint64_t t1 = lad::dev::globaltimer_ns();
            while (!mbar_try_wait(mbar_a, static_cast<uint32_t>(p.nseg) & 1u) &&
                   lad::dev::globaltimer_ns() - t1 < lad::dev::kWaitLimitNs) {
            }
        }
        __syncwarp();
    }
    if (tid == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kCTmemCols);
}

}  // namespace

namespace lad {
int take_device_error_prefill(cudaStream_t s, int *code) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_prefill_error, sizeof v, 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return set_error(LAD_ECUDA, "lad_device_error: %s", cudaGetErrorString(e));
    if (v) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_prefill_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return set_error(LAD_ECUDA, "lad_device_error: %s", cudaGetErrorString(e));
    }
    *code = v;
    return LAD_OK;
}
}  // namespace lad

namespace {
// The split path's workspace: a header of per-segment item counters (256-byte granules), then one
// segment buffer of records, or two when there are several segments (the prep of segment s + 1
// writes one while the chain of segment s reads the other).
// With several segments the last one is short (kTailChunks): its chain is the one piece of work
// that nothing overlaps, so it should be brief; the segments before it hold up to kSegChunks.
constexpr int kTailChunks = 32;
struct WsLayout {
    long long nch, head, seg, nsegs, nbuf, header, buf_bytes;
    bool tail(long long k) const { return nsegs > 1 && k == nsegs - 1; }
    long long first(long long k) const { return tail(k) ? head : k * seg; }  // segment k's first chunk
    long long count(long long k) const {
        if (nsegs == 1) return nch;
        return tail(k) ? nch - head : (seg < head - first(k) ? seg : head - first(k));
    }
};
WsLayout ws_layout(int B, int T, int H) {
    WsLayout L;
    L.nch = (static_cast<long long>(T) + kC - 1) / kC;
    if (L.nch <= kSegChunks) {
        L.seg = L.head = L.nch;
        L.nsegs = 1;
    } else {
        L.seg = kSegChunks;
        L.head = L.nch - kTailChunks;                 // chunks before the tail segment
        L.nsegs = (L.head + L.seg - 1) / L.seg + 1;  // the last of these starts at chunk `head`
    }
    L.nbuf = L.nsegs > 1 ? 2 : 1;
    L.header = (L.nsegs * 4 + 255) / 256 * 256;
    L.buf_bytes = static_cast<long long>(B) * H * L.seg * kRecBytes;
    return L;
}

// Per device: the stream the chain kernels run on, at the highest priority (when SMs free up, a
// chain launch is placed ahead of the next segment's prep CTAs), and the events that order the two
// streams. The mutex also serialises a call's whole enqueue sequence, as the events are shared.
struct SideStream {
    cudaStream_t st = nullptr;
    cudaEvent_t prep_done = nullptr, chain_done[2] = {nullptr, nullptr};
};
std::mutex side_mu;
SideStream side_streams[64];

cudaError_t side_stream(int dev, SideStream **out) {
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    SideStream &s = side_streams[dev];
    if (!s.st) {
        int least = 0, greatest = 0;
        cudaError_t e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
        if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&s.st, cudaStreamNonBlocking, greatest);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.prep_done, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.chain_done[0], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.chain_done[1], cudaEventDisableTiming);
        if (e != cudaSuccess) {
            s = SideStream{};  // handles created before the failure stay alive; nothing reuses them
            return e;
        }
    }
    *out = &s;
    return cudaSuccess;
}
}  // namespace

extern "C" size_t kda_prefill_workspace_size(int B, int T, int H, int dk, int dv, int chunk) {
    if (B <= 0 || T <= 0 || H <= 0 || dk != kDk || dv != kDv || chunk != kC) return 0;
    const WsLayout L = ws_layout(B, T, H);
    return static_cast<size_t>(L.header + L.nbuf * L.buf_bytes);
}

extern "C" int kda_prefill_chunked(const lad_bf16 *q, const lad_bf16 *k, const lad_bf16 *v, const float *alpha,
                                   const float *beta, float *S, void *o, int B, int T, int H, int dk, int dv,
                                   int chunk, float scale, unsigned flags, void *workspace, size_t ws_bytes,
                                   void *stream) {
    using lad::set_error;
    if (B < 0 || T < 0 || H < 0) return set_error(LAD_EINVAL, "kda_prefill_chunked: negative size");
    if (dk != kDk || dv != kDv) return set_error(LAD_EUNSUPPORTED, "kda_prefill_chunked: dk = dv = 128 only");
    if (chunk != kC) return set_error(LAD_EUNSUPPORTED, "kda_prefill_chunked: chunk = 64 only");
    if (flags & ~(LAD_FLAG_OUT_FP32 | LAD_FLAG_L2NORM_QK))
        return set_error(LAD_EINVAL, "kda_prefill_chunked: unknown flags 0x%x", flags);
    if (B == 0 || H == 0) return LAD_OK;
    if (!S) return set_error(LAD_EINVAL, "kda_prefill_chunked: null S");
    if (T == 0) return LAD_OK;  // the state passes through unchanged
    if (!q || !k || !v || !alpha || !beta || !o) return set_error(LAD_EINVAL, "kda_prefill_chunked: null pointer");
    const bool f32 = (flags & LAD_FLAG_OUT_FP32) != 0;
    if (!lad::aligned(S, 16) || !lad::aligned(v, 16) || !lad::aligned(o, 16) || !lad::aligned(q, 16) ||
        !lad::aligned(k, 16) || !lad::aligned(alpha, 16))
        return set_error(LAD_EUNSUPPORTED, "kda_prefill_chunked: q, k, v, alpha, S and o must be 16-byte aligned");
    const long long ctas = 2LL * B * H;
    if (ctas > 0x7fffffffLL) return set_error(LAD_EUNSUPPORTED, "kda_prefill_chunked: B*H too large");
    const size_t ws_need = kda_prefill_workspace_size(B, T, H, dk, dv, chunk);
    const bool split = workspace != nullptr;
    if (split && (ws_bytes < ws_need || !lad::aligned(workspace, 256)))
        return set_error(LAD_EWORKSPACE, "kda_prefill_chunked: workspace of %zu bytes (256-byte aligned) required, or NULL",
                         ws_need);
    if (split && static_cast<long long>(B) * H * kSegChunks > 0x7fffffffLL)
        return set_error(LAD_EUNSUPPORTED, "kda_prefill_chunked: B*H too large");
    {
        // the dynamic shared memory limits, set once per device
        static std::mutex attr_mu;
        static bool attr_done[64] = {};
        int adev = 0;
        if (cudaGetDevice(&adev) != cudaSuccess || adev < 0 || adev >= 64)
            return set_error(LAD_ECUDA, "kda_prefill_chunked: no current device");
        std::lock_guard<std::mutex> lock(attr_mu);
        if (!attr_done[adev]) {
            cudaError_t attr_err =
                cudaFuncSetAttribute(kda_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            if (attr_err == cudaSuccess)
                attr_err = cudaFuncSetAttribute(kda_chunk_prep_ws_kernel<false>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, kWSmemBytes);
            if (attr_err == cudaSuccess)
                attr_err = cudaFuncSetAttribute(kda_chunk_prep_ws_kernel<true>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, kWSmemBytes);
            if (attr_err == cudaSuccess)
                attr_err = cudaFuncSetAttribute(kda_chunk_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                kCSmemBytes);
            if (attr_err != cudaSuccess)
                return set_error(LAD_ECUDA, "kda_prefill_chunked: smem attribute: %s", cudaGetErrorString(attr_err));
            attr_done[adev] = true;
        }
    }
    Args a{reinterpret_cast<const uint16_t *>(q), reinterpret_cast<const uint16_t *>(k),
           reinterpret_cast<const uint16_t *>(v), alpha, beta, S, o, B, T, H, scale,
           (flags & LAD_FLAG_L2NORM_QK) ? 1 : 0, f32 ? 1 : 0};
    auto enc = reinterpret_cast<EncodeTiledFn>(lad::tensor_map_encoder_raw());
    if (!enc) return set_error(LAD_ECUDA, "kda_prefill_chunked: cuTensorMapEncodeTiled unavailable");
    auto make = [&](CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, int box0, bool sw128,
                    int box1 = kC) -> int {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(H) * kDk, static_cast<cuuint64_t>(T),
                                    static_cast<cuuint64_t>(B)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(H) * kDk * esize,
                                       static_cast<cuuint64_t>(T) * H * kDk * esize};
        const cuuint32_t box[3] = {static_cast<cuuint32_t>(box0), static_cast<cuuint32_t>(box1), 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         sw128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        return r == CUDA_SUCCESS ? LAD_OK : set_error(LAD_ECUDA, "kda_prefill_chunked: tensor map failed (%d)", (int)r);
    };
    cudaStream_t st = lad::as_stream(stream);
    if (!split) {
        Maps maps;
        int rc = make(&maps.q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDk, false);
        if (rc == LAD_OK) rc = make(&maps.k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDk, false);
        if (rc == LAD_OK) rc = make(&maps.alpha, alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kDk, false);
        if (rc == LAD_OK) rc = make(&maps.v, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDvh, false);
        if (rc != LAD_OK) return rc;
        kda_prefill_kernel<<<static_cast<unsigned>(ctas), kThreads, kSmemBytes, st>>>(a, maps);
        return lad::check_launch("kda_prefill_chunked");
    }
    // split path, segment by segment: every chunk's operands of the segment (prep), then the chain
    PrepMaps pm;
    int rc = make(&pm.q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDk, false);
    if (rc == LAD_OK) rc = make(&pm.k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDk, false);
    if (rc == LAD_OK) rc = make(&pm.alpha, alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kDk, false);
    ChainMaps cm;
    if (rc == LAD_OK)
        rc = make(&cm.o, o, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 ? 4 : 2, kDv,
                  false, f32 ? kC / 2 : kC);
    if (rc == LAD_OK) rc = make(&cm.v, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64, true);
    if (rc != LAD_OK) return rc;
    const WsLayout L = ws_layout(B, T, H);
    const int sms = lad::device_sm_count();
    if (sms <= 0) return set_error(LAD_ECUDA, "kda_prefill_chunked: cannot query the SM count");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return set_error(LAD_ECUDA, "kda_prefill_chunked: no current device");
    std::lock_guard<std::mutex> lock(side_mu);
    SideStream *side = nullptr;
    cudaError_t e = side_stream(dev, &side);
    if (e != cudaSuccess) return set_error(LAD_ECUDA, "kda_prefill_chunked: side stream: %s", cudaGetErrorString(e));
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *counters = reinterpret_cast<int *>(ws);
    e = cudaMemsetAsync(counters, 0, static_cast<size_t>(L.header), st);
    // Segment s: its prep, then its chain on the side stream. The prep of s + 1 runs beside the chain
    // of s: `beside` CTAs on the caller's stream take the SMs the chain leaves (a launch that
    // could take every SM would be placed first and hold them all, the chain waiting behind it),
    // and the rest join on the side stream as soon as the chain is done, from the same item
    // counter. The prep of s + 2 waits for the chain of s to free its buffer.
    const int chain_ctas = B * H < sms ? B * H : sms;
    const int beside = sms - chain_ctas > sms / 2 ? sms - chain_ctas : sms / 2;
    auto prep = [&](cudaStream_t on, long long grid, int sg, uint8_t *buf, int c0, int nseg) {
        const PrepArgs pa{beta, buf, counters + sg, B, T, H, c0, nseg, a.l2norm};
        if (a.l2norm)
            kda_chunk_prep_ws_kernel<true><<<static_cast<unsigned>(grid), kPThreads, kWSmemBytes, on>>>(pa, pm);
        else
            kda_chunk_prep_ws_kernel<false><<<static_cast<unsigned>(grid), kPThreads, kWSmemBytes, on>>>(pa, pm);
        return cudaGetLastError();
    };
    for (int sg = 0; sg < L.nsegs && e == cudaSuccess; ++sg) {
        const int c0 = static_cast<int>(L.first(sg));
        const int nseg = static_cast<int>(L.count(sg));
        uint8_t *buf = ws + L.header + (sg % L.nbuf) * L.buf_bytes;
        const long long items = static_cast<long long>(B) * H * nseg;
        if (sg == 0) {
            e = prep(st, items < sms ? items : sms, sg, buf, c0, nseg);
        } else {
            if (sg >= 2) e = cudaStreamWaitEvent(st, side->chain_done[sg & 1], 0);
            if (e == cudaSuccess) e = prep(st, items < beside ? items : beside, sg, buf, c0, nseg);
            if (e == cudaSuccess) e = prep(side->st, items < sms - beside ? items : sms - beside, sg, buf, c0, nseg);
        }
        if (e == cudaSuccess) e = cudaEventRecord(side->prep_done, st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(side->st, side->prep_done, 0);
        if (e != cudaSuccess) break;
        kda_chunk_chain_kernel<<<static_cast<unsigned>(B * H), kChainThreads, kCSmemBytes, side->st>>>(
            ChainArgs{S, o, buf, B, T, H, c0, nseg, scale, a.out_f32}, cm);
        e = cudaGetLastError();
        if (e == cudaSuccess) e = cudaEventRecord(side->chain_done[sg & 1], side->st);
    }
    // the caller's stream waits for the last chain (when the loop stopped early, for whatever was
    // enqueued on the side stream)
    const cudaError_t j = cudaStreamWaitEvent(st, side->chain_done[(L.nsegs - 1) & 1], 0);
    if (e == cudaSuccess) e = j;
    if (e != cudaSuccess) return set_error(LAD_ECUDA, "kda_prefill_chunked: %s", cudaGetErrorString(e));
    return LAD_OK;
}
