// KDA chunked prefill on B200: the gated delta rule over T tokens in chunks of 64, in the WY / UT
// form, with every contraction on the tensor cores (tcgen05, kind::tf32) and the fp32 state
// carried in tensor memory from chunk to chunk.
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
// d_v columns of S are independent, so a CTA owns one (sequence, head, half of d_v) and walks
// its chunks in order: 128 CTAs for one sequence of 64 heads.
//
// Two paths. With a workspace, two kernels per segment of up to 128 chunks: the prep kernel
// computes every chunk's state-independent operands (W, Tb V, Qt, Kh^T, lower(Qt Kh^T), g_last)
// in parallel into a record per chunk, and the scan kernel runs only the state chain, two MMA
// batches per chunk (see "Split path" below). Without one, the single kernel does both, per chunk:
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
// Split path: the chunk-local, state-independent part of every chunk in parallel (prep), then
// the state chain alone (scan). With S0 the state entering a chunk:
//   X = W S0,  O = scale (Qt S0 + P (U' - X)),  S = Diag(g_last) (S0 + Kh^T (U' - X))
// where W = Tb Kt, U' = Tb V and P = lower(Qt Kh^T) depend only on the chunk's own inputs. The
// scan then runs two MMA batches per chunk instead of three, and none of the chunk's operand
// formation or the (I + A)^-1 solve stays on the serial chain; the price is the per-chunk
// operands' round trip through HBM (one record per (sequence, head, chunk)).
// ------------------------------------------------------------------------------------------

// Record of one (sequence, head, chunk) in the workspace. The four tiles are stored exactly as
// their shared-memory operand tiles (K-major, tf32-rounded fp32, 128-byte swizzle, 1 KiB aligned),
// so the scan copies them byte for byte.
constexpr uint32_t kItW = 0;          // W = Tb Kt [64 tok][128 d_k]: 4 blocks x 8 KiB
constexpr uint32_t kItQ = 32768;      // Qt [64 tok][128 d_k]: 4 blocks x 8 KiB
constexpr uint32_t kItKHT = 65536;    // Kh^T [128 d_k][64 tok]: 2 blocks x 16 KiB
constexpr uint32_t kItP = 98304;      // lower(Qt Kh^T) [64][64]: 2 blocks x 8 KiB
constexpr uint32_t kItU = 114688;     // U' = Tb V, plain fp32 [2 d_v halves][64 tok][64]
constexpr uint32_t kItG = 147456;     // g_last [128] fp32
constexpr uint32_t kItemBytes = 148480;  // 145 KiB
constexpr int kSegChunks = 128;          // chunks per segment (prep then scan), bounds the workspace

// prep shared memory
constexpr uint32_t kPStA = 0, kPStQ = 32768, kPStK = 49152, kPStV = 65536;  // raw staging (80 KiB)
constexpr uint32_t kPKHT = 0;        // Kh^T [128][64], stride 16 KiB (over the staged alpha)
constexpr uint32_t kPKTT = 32768;    // Kt^T [128][64], stride 16 KiB (over the staged q, k)
constexpr uint32_t kPP = 65536;      // P [64][64], stride 8 KiB (over the staged v)
constexpr uint32_t kPXQK = 81920;    // [Qt; Kt] 128 x 128, stride 16 KiB
constexpr uint32_t kPTT = kPXQK + 8192;  // Tb in the Kt half of XQK blocks 0-1
constexpr uint32_t kPKH = 147456;    // Kh [64][128], stride 8 KiB; then the A / T scratch
constexpr uint32_t kPVT = 180224;    // V^T [128 d_v][64 tok], stride 16 KiB
constexpr uint32_t kPMisc = 212992;
constexpr uint32_t kPStageTx = 32768 + 16384 + 16384 + 16384;
constexpr uint32_t kPSmemBytes = kPMisc + kMiscOct + 8 * 128 * 4 + 1024;

constexpr uint32_t kPColAcc1 = 0;    // M=128 x 64: [Qt Kh^T ; Kt Kh^T]
constexpr uint32_t kPColW = 64;      // M=64 x 128: W = Tb Kt
constexpr uint32_t kPColU = 192;     // M=64 x 128: U' = Tb V
constexpr uint32_t kIdesc64x128 = make_idesc(64, 128, kFmtTf32, 0, 0);

struct SplitArgs {
    const uint16_t *q, *k, *v;
    const float *alpha, *beta;
    float *S;
    void *o;
    uint8_t *ws;        // records of this segment, [B*H][nseg]
    int B, T, H;
    int c0, nseg;       // the segment: chunks c0 .. c0 + nseg - 1
    float scale;
    int l2norm, out_f32;
};

// Bulk copy shared -> global by one thread, in the thread's current bulk group; both addresses
// 16-byte aligned, bytes a multiple of 16. The shared source must not change until
// bulk_wait_read has seen the group through.
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(reinterpret_cast<uint64_t>(dst)),
                 "r"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {  // all but the newest N groups have read their source
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// One CTA per SM walks the segment's (sequence, head, chunk) items; the next item's raw inputs are
// staged (alpha once Kh^T has been written out, q, k, v once the second MMA batch is complete).
__global__ void __launch_bounds__(kThreads, 1) kda_prefill_prep_kernel(SplitArgs p,
                                                                      const __grid_constant__ Maps maps) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    float *s_beta = reinterpret_cast<float *>(sm + kPMisc + kMiscBeta);
    float *s_rq = reinterpret_cast<float *>(sm + kPMisc + kMiscRq);
    float *s_rk = reinterpret_cast<float *>(sm + kPMisc + kMiscRk);
    float *s_gc = reinterpret_cast<float *>(sm + kPMisc + kMiscGc);
    float *s_oct = reinterpret_cast<float *>(sm + kPMisc + kMiscOct);
    const uint32_t bar = sbase + kPMisc + kMiscBar;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kPMisc + kMiscTmem);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kPMisc + kMiscAbort);
    const uint32_t tma_bar = sbase + kPMisc + kMiscTmaBar;
    float *Apl = reinterpret_cast<float *>(sm + kPKH);
    float *Tpl = reinterpret_cast<float *>(sm + kPKH + 64 * 64 * 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = warp & 3, cg = warp >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(32 * sp) << 16;
    const int row128 = 32 * sp + lane;
    const int row64 = 16 * sp + lane;
    const uint64_t d0 = smem_desc(sbase, 16, 1024, kLayoutSw128);
    const int nitems = p.B * p.H * p.nseg;

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
    uint32_t phase = 0, tma_phase = 0;
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
    // item -> (b, h, chunk); items of one (b, h) are consecutive
    auto coords = [&](int item, int &b, int &h, int &ch) {
        const int bh = item / p.nseg;
        ch = p.c0 + (item - bh * p.nseg);
        b = bh / p.H;
        h = bh - b * p.H;
    };
    auto stage_alpha = [&](int item) {
        int b, h, ch;
        coords(item, b, h, ch);
        fence_async_smem();
        mbar_arrive_tx_raw(tma_bar, kPStageTx);
        tma_load_3d(sbase + kPStA, &maps.alpha, h * kDk, ch * kC, b, tma_bar);
    };
    auto stage_qkv = [&](int item) {
        int b, h, ch;
        coords(item, b, h, ch);
        fence_async_smem();
        tma_load_3d(sbase + kPStQ, &maps.q, h * kDk, ch * kC, b, tma_bar);
        tma_load_3d(sbase + kPStK, &maps.k, h * kDk, ch * kC, b, tma_bar);
        tma_load_3d(sbase + kPStV, &maps.v, h * kDv, ch * kC, b, tma_bar);
    };
    int pending = 0, qkv_owed = -1;
    int item = blockIdx.x;
    if (item < nitems) {
        if (tid == 0) {
            stage_alpha(item);
            stage_qkv(item);
        }
        pending = 1;
    }
    for (; item < nitems && ok; item += gridDim.x) {
        int b, h, ch;
        coords(item, b, h, ch);
        const int next = item + static_cast<int>(gridDim.x);
        const int t0 = ch * kC;
        const int n = min(kC, p.T - t0);
        const size_t tok0 = (static_cast<size_t>(b) * p.T + t0) * p.H + h;
        const size_t tstride = static_cast<size_t>(p.H);
        uint8_t *rec = p.ws + static_cast<size_t>(item) * kItemBytes;

        if (tid < kC) s_beta[tid] = (tid < n) ? p.beta[tok0 + tid * tstride] : 0.f;
        if (tid == 0) bulk_wait_read<0>();  // the previous item's W and U' have left [Qt; Kt]
        {
            const bool w = wait_bar(tma_bar, tma_phase, abort_flag, &g_prefill_error, lad::kErrPrefill);
            tma_phase ^= 1;
            pending = 0;
            ok = __syncthreads_and(w) != 0;
            if (!ok) break;
        }
        if (p.l2norm) {
            const uint16_t *sq = reinterpret_cast<const uint16_t *>(sm + kPStQ);
            const uint16_t *sk = reinterpret_cast<const uint16_t *>(sm + kPStK);
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

        // ---- running decay and the operand tiles (warp w: tokens 8w..8w+7; lane l: channels 4l..) ----
        {
            const int o = warp, c4 = 4 * lane;
            const float *sa = reinterpret_cast<const float *>(sm + kPStA);
            const uint16_t *sq = reinterpret_cast<const uint16_t *>(sm + kPStQ);
            const uint16_t *sk = reinterpret_cast<const uint16_t *>(sm + kPStK);
            float4 gl[8];
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
            float4 excl = make_float4(1.f, 1.f, 1.f, 1.f);
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
                st_tile4(sm + kPXQK, r, c4, kStr16, qv[0] * gg[0], qv[1] * gg[1], qv[2] * gg[2], qv[3] * gg[3]);
                st_tile4(sm + kPXQK, kC + r, c4, kStr16, kv[0] * gg[0], kv[1] * gg[1], kv[2] * gg[2], kv[3] * gg[3]);
                st_tile4(sm + kPKH, r, c4, kStr8, __fdividef(kv[0], gg[0]), __fdividef(kv[1], gg[1]),
                         __fdividef(kv[2], gg[2]), __fdividef(kv[3], gg[3]));
            }
            // V^T [128 d_v][64 tok]: thread -> value column j = tid % 128, tokens 32 * (tid / 128) .. + 31
            const uint16_t *sv = reinterpret_cast<const uint16_t *>(sm + kPStV);
            const int j = tid & 127, r0 = 32 * (tid >> 7);
#pragma unroll 2
            for (int r = 0; r < 32; r += 4)
                st_tile4(sm + kPVT, j, r0 + r, kStr16, bf16_to_f32(sv[(r0 + r) * kDv + j]),
                         bf16_to_f32(sv[(r0 + r + 1) * kDv + j]), bf16_to_f32(sv[(r0 + r + 2) * kDv + j]),
                         bf16_to_f32(sv[(r0 + r + 3) * kDv + j]));
        }
        // ---- MMA 1: [Qt; Kt] Kh^T, issued now; the transposes below only read its operands ----
        fence_async_smem();
        tc_fence_before();
        __syncthreads();  // the staging area is read: Kh^T and Kt^T go over it
        if (warp == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < kDk / 8; ++j)
                tc_mma_tf32(tmem + kPColAcc1, kdesc(d0 + (kPXQK >> 4), kStr16, j), kdesc(d0 + (kPKH >> 4), kStr8, j),
                            kIdesc128, j > 0);
            tc_commit(bar);
        }
        {
            // Kh^T from Kh, Kt^T from the Kt rows of [Qt; Kt]: thread -> channel i, tokens of half th
            const int i = tid & (kDk - 1), th = tid >> 7;
#pragma unroll 2
            for (int r = (kC / 2) * th; r < (kC / 2) * (th + 1); r += 4) {
                float kh[4], kt[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    kh[u] = *reinterpret_cast<const float *>(sm + kPKH + sw128_off32(r + u, i, kStr8));
                    kt[u] = *reinterpret_cast<const float *>(sm + kPXQK + sw128_off32(kC + r + u, i, kStr16));
                }
                st_tile4(sm + kPKHT, i, r, kStr16, kh[0], kh[1], kh[2], kh[3]);
                st_tile4(sm + kPKTT, i, r, kStr16, kt[0], kt[1], kt[2], kt[3]);
            }
        }
        fence_async_smem();  // the transposes are read by the bulk store below
        {
            const bool w = wait_bar(bar, phase, abort_flag, &g_prefill_error, lad::kErrPrefill);
            phase ^= 1;
            tc_fence_after();
            ok = __syncthreads_and(w) != 0;
            if (!ok) break;
        }
        // Kh^T, Qt and g_last are final: out to the record by bulk stores (group 1)
        if (tid == 0) {
            bulk_s2g(rec + kItKHT, sbase + kPKHT, 32768);
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) bulk_s2g(rec + kItQ + blk * 8192, sbase + kPXQK + blk * kStr16, 8192);
            bulk_s2g(rec + kItG, smem_u32(s_gc), 512);
            bulk_commit();
        }
        // ---- lower(Qt Kh^T) -> P tile (rows 0-63); A = strict_lower(diag(beta) Kt Kh^T) -> scratch ----
        {
            float x[32];
            tmem_ld32(tmem + lane_base + kPColAcc1 + 32 * cg, x);
            tmem_wait_ld();
            const int c0 = 32 * cg;
            if (row128 < kC) {
                const int r = row128;
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    st_tile4(sm + kPP, r, c0 + j, kStr8, c0 + j <= r ? x[j] : 0.f, c0 + j + 1 <= r ? x[j + 1] : 0.f,
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
        }
        fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            bulk_s2g(rec + kItP, sbase + kPP, 16384);  // group 2
            bulk_commit();
            bulk_wait_read<1>();  // group 1 has read Kh^T: the next item's alpha can come in over it
        }
        if (next < nitems) {
            if (tid == 0) stage_alpha(next);
            pending = 1;
            qkv_owed = next;
        }
        // ---- T = (I + A)^-1, Tb -> operand ----
        solve_tb(Apl, Tpl, s_beta, sm + kPTT, tid);
        // ---- MMA 2: W = Tb Kt (B = Kt^T), U' = Tb V (B = V^T) ----
        ok = mma_sync([&] {
#pragma unroll
            for (int j = 0; j < kC / 8; ++j) {
                const uint64_t tt = kdesc(d0 + (kPTT >> 4), kStr16, j);
                tc_mma_tf32(tmem + kPColW, tt, kdesc(d0 + (kPKTT >> 4), kStr16, j), kIdesc64x128, j > 0);
                tc_mma_tf32(tmem + kPColU, tt, kdesc(d0 + (kPVT >> 4), kStr16, j), kIdesc64x128, j > 0);
            }
        });
        if (!ok) break;
        if (tid == 0) bulk_wait_read<0>();  // P (and Qt) read out: the staging area and XQK are free
        if (qkv_owed >= 0) {  // Kt^T and P are done with: q, k, v of the next item
            if (tid == 0) stage_qkv(qkv_owed);
            qkv_owed = -1;
        }
        __syncthreads();
        // ---- W (tf32-rounded operand layout) and U' (plain fp32, per d_v half) -> shared memory over
        //      [Qt; Kt], then -> record by one bulk store (group 3) ----
        {
            float *ush = reinterpret_cast<float *>(sm + kPXQK + 32768);  // U' [2 halves][64 tok][64]
#pragma unroll 1
            for (int part = 0; part < 2; ++part) {
                const int c0 = 32 * cg + 64 * part;  // columns c0 .. c0 + 31
                float w[32], u[32];
                tmem_ld32(tmem + lane_base + kPColW + c0, w);
                tmem_ld32(tmem + lane_base + kPColU + c0, u);
                tmem_wait_ld();
                if (lane < 16) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        st_tile4(sm + kPXQK, row64, c0 + j, kStr8, w[j], w[j + 1], w[j + 2], w[j + 3]);
                        const int hv = c0 >> 6, cc = (c0 & 63) + j;
                        *reinterpret_cast<float4 *>(ush + (hv * 64 + row64) * 64 + cc) =
                            make_float4(u[j], u[j + 1], u[j + 2], u[j + 3]);
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            bulk_s2g(rec + kItW, sbase + kPXQK, 32768);
            bulk_s2g(rec + kItU, sbase + kPXQK + 32768, 32768);
            bulk_commit();
        }
    }
    if (tid == 0 && qkv_owed >= 0) stage_qkv(qkv_owed);
    if (tid == 0 && pending) {
        const uint64_t t0 = lad::dev::globaltimer_ns();
        while (!mbar_try_wait(tma_bar, tma_phase) && lad::dev::globaltimer_ns() - t0 < lad::dev::kWaitLimitNs) {
        }
    }
    if (tid == 0) bulk_wait_all();  // every record write has landed
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

// scan shared memory: W and Qt (single buffer), then two buffers of Kh^T, P and g_last (the
// second batch's operands arrive a whole chunk ahead), S0^T, U^T; U' goes straight to registers
constexpr uint32_t kSW = 0, kSQ = 32768;
constexpr uint32_t kSKP0 = 65536, kSKPBytes = 50176;  // a buffer: Kh^T 32 KiB, P 16 KiB, g_last 512 B (+pad)
constexpr uint32_t kSKHT = 0, kSP = 32768, kSG = 49152;  // offsets inside a buffer
constexpr uint32_t kSSOT = kSKP0 + 2 * kSKPBytes;   // 165,888: S0^T [64 d_v][128 d_k], stride 8 KiB
constexpr uint32_t kSUT = kSSOT + 32768;            // U^T [64 d_v][64 tok], stride 8 KiB
constexpr uint32_t kSMisc = kSUT + 16384;           // bars, tmem slot, abort flag
constexpr uint32_t kSSmemBytes = kSMisc + 2048 + 1024;
constexpr uint32_t kSBar1Tx = 65536;                // W, Qt
constexpr uint32_t kSBar2Tx = 32768 + 16384 + 512;  // Kh^T, P, g_last
constexpr uint32_t kSColX = 0, kSColO = 64, kSColS = 128;
constexpr uint32_t kSTmemCols = 256;

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// One CTA per (sequence, head, half of d_v) walks the segment's chunks with the state in TMEM.
__global__ void __launch_bounds__(kThreads, 1) kda_prefill_scan_kernel(SplitArgs p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const uint32_t bar = sbase + kSMisc;
    const uint32_t bar1 = sbase + kSMisc + 8;
    auto bar2 = [&](int j) { return sbase + kSMisc + 16 + 8u * static_cast<uint32_t>(j); };  // per buffer
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kSMisc + 32);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kSMisc + 36);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = warp & 3, cg = warp >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(32 * sp) << 16;
    const int row128 = 32 * sp + lane;
    const int row64 = 16 * sp + lane;
    const int half = blockIdx.x & 1;
    const int bh = blockIdx.x >> 1;
    const int b = bh / p.H, h = bh - b * p.H;
    const uint64_t d0 = smem_desc(sbase, 16, 1024, kLayoutSw128);
    const uint8_t *recs = p.ws + static_cast<size_t>(bh) * p.nseg * kItemBytes;

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar1, 1);
        mbar_init(bar2(0), 1);
        mbar_init(bar2(1), 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kSTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t phase = 0, ph1 = 0, ph2[2] = {0, 0};
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
    auto load1 = [&](int i) {  // W, Qt of chunk i of the segment
        const uint8_t *rec = recs + static_cast<size_t>(i) * kItemBytes;
        fence_async_smem();
        mbar_arrive_tx_raw(bar1, kSBar1Tx);
        bulk_g2s(sbase + kSW, rec + kItW, 32768, bar1);
        bulk_g2s(sbase + kSQ, rec + kItQ, 32768, bar1);
    };
    auto load2 = [&](int i) {  // Kh^T, P, g_last of chunk i into buffer i % 2
        const uint8_t *rec = recs + static_cast<size_t>(i) * kItemBytes;
        const uint32_t buf = sbase + kSKP0 + (i & 1) * kSKPBytes;
        fence_async_smem();
        mbar_arrive_tx_raw(bar2(i & 1), kSBar2Tx);
        bulk_g2s(buf + kSKHT, rec + kItKHT, 32768, bar2(i & 1));
        bulk_g2s(buf + kSP, rec + kItP, 16384, bar2(i & 1));
        bulk_g2s(buf + kSG, rec + kItG, 512, bar2(i & 1));
    };
    int pend1 = 0, pend2[2] = {0, 0};
    if (tid == 0) {
        load1(0);
        load2(0);
        if (p.nseg > 1) load2(1);
    }
    pend1 = pend2[0] = 1;
    pend2[1] = p.nseg > 1 ? 1 : 0;

    // ---- the state entering the segment: TMEM master (row = key channel) and the S0^T operand ----
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
        for (int j = 0; j < 32; ++j) st_tile1(sm + kSSOT, 32 * cg + j, row128, kStr8, v[j]);
        tmem_st32(tmem + lane_base + kSColS + 32 * cg, v);
        tmem_wait_st();
    }

    for (int i = 0; i < p.nseg && ok; ++i) {
        const int ch = p.c0 + i;
        const int t0 = ch * kC;
        const int n = min(kC, p.T - t0);
        const size_t tok0 = (static_cast<size_t>(b) * p.T + t0) * p.H + h;
        const size_t tstride = static_cast<size_t>(p.H);
        // this chunk's U' (rows of this thread, 32 of this CTA's d_v columns) straight into registers
        float4 up[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) up[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lane < 16) {  // rows 0-63 of the M = 64 accumulator sit in lanes 0-15
            const float4 *src = reinterpret_cast<const float4 *>(recs + static_cast<size_t>(i) * kItemBytes + kItU +
                                                                 half * 16384) +
                                (row64 * 64 + 32 * cg) / 4;
#pragma unroll
            for (int j = 0; j < 8; ++j) up[j] = src[j];
        }
        {
            const bool w = wait_bar(bar1, ph1, abort_flag, &g_prefill_error, lad::kErrPrefill);
            ph1 ^= 1;
            pend1 = 0;
            ok = __syncthreads_and(w) != 0;
            if (!ok) break;
        }
        // ---- X = W S0,  O = Qt S0 ----
        ok = mma_sync([&] {
#pragma unroll
            for (int j = 0; j < kDk / 8; ++j) {
                const uint64_t sot = kdesc(d0 + (kSSOT >> 4), kStr8, j);
                tc_mma_tf32(tmem + kSColX, kdesc(d0 + (kSW >> 4), kStr8, j), sot, kIdesc64, j > 0);
                tc_mma_tf32(tmem + kSColO, kdesc(d0 + (kSQ >> 4), kStr8, j), sot, kIdesc64, j > 0);
            }
        });
        if (!ok) break;
        if (i + 1 < p.nseg) {
            if (tid == 0) load1(i + 1);
            pend1 = 1;
        }
        const int kb = i & 1;
        const uint32_t kp = kSKP0 + static_cast<uint32_t>(kb) * kSKPBytes;
        {
            const bool w = wait_bar(bar2(kb), ph2[kb], abort_flag, &g_prefill_error, lad::kErrPrefill);
            ph2[kb] ^= 1;
            pend2[kb] = 0;
            ok = __syncthreads_and(w) != 0;
            if (!ok) break;
        }
        const float gc = reinterpret_cast<const float *>(sm + kp + kSG)[row128];
        // ---- U = U' - X -> U^T operand ----
        {
            float x[32];
            tmem_ld32(tmem + lane_base + kSColX + 32 * cg, x);
            tmem_wait_ld();
            if (lane < 16) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    st_tile1(sm + kSUT, 32 * cg + 4 * j, row64, kStr8, up[j].x - x[4 * j]);
                    st_tile1(sm + kSUT, 32 * cg + 4 * j + 1, row64, kStr8, up[j].y - x[4 * j + 1]);
                    st_tile1(sm + kSUT, 32 * cg + 4 * j + 2, row64, kStr8, up[j].z - x[4 * j + 2]);
                    st_tile1(sm + kSUT, 32 * cg + 4 * j + 3, row64, kStr8, up[j].w - x[4 * j + 3]);
                }
            }
        }
        // ---- O += P U;  S += Kh^T U ----
        ok = mma_sync([&] {
#pragma unroll
            for (int j = 0; j < kC / 8; ++j) {
                const uint64_t ut = kdesc(d0 + (kSUT >> 4), kStr8, j);
                tc_mma_tf32(tmem + kSColO, kdesc(d0 + ((kp + kSP) >> 4), kStr8, j), ut, kIdesc64, 1);
                tc_mma_tf32(tmem + kSColS, kdesc(d0 + ((kp + kSKHT) >> 4), kStr16, j), ut, kIdesc128, 1);
            }
        });
        if (!ok) break;
        if (i + 2 < p.nseg) {  // this buffer is free again: chunk i + 2's operands
            if (tid == 0) load2(i + 2);
            pend2[kb] = 1;
        }
        // ---- O -> HBM; S <- Diag(g_last) S, S^T -> operand (HBM after the segment's last chunk) ----
        {
            float ov[32];
            tmem_ld32(tmem + lane_base + kSColO + 32 * cg, ov);
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
            float sv[32];
            tmem_ld32(tmem + lane_base + kSColS + 32 * cg, sv);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                sv[j] *= gc;
                st_tile1(sm + kSSOT, 32 * cg + j, row128, kStr8, sv[j]);
            }
            tmem_st32(tmem + lane_base + kSColS + 32 * cg, sv);
            if (i == p.nseg - 1) {
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
    // drain: copies still in flight (after an abort) land, MMAs complete, before release
    if (tid == 0) {
        const uint64_t t0 = lad::dev::globaltimer_ns();
        while (pend1 && !mbar_try_wait(bar1, ph1) && lad::dev::globaltimer_ns() - t0 < lad::dev::kWaitLimitNs) {
        }
        for (int j = 0; j < 2; ++j)
            while (pend2[j] && !mbar_try_wait(bar2(j), ph2[j]) &&
                   lad::dev::globaltimer_ns() - t0 < lad::dev::kWaitLimitNs) {
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
    if (warp == 0) tmem_dealloc(tmem, kSTmemCols);
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

extern "C" size_t kda_prefill_workspace_size(int B, int T, int H, int dk, int dv, int chunk) {
    if (B <= 0 || T <= 0 || H <= 0 || dk != kDk || dv != kDv || chunk != kC) return 0;
    const long long nch = (static_cast<long long>(T) + kC - 1) / kC;
    const long long seg = nch < kSegChunks ? nch : kSegChunks;
    return static_cast<size_t>(B) * static_cast<size_t>(H) * static_cast<size_t>(seg) * kItemBytes;
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
    if (split && (ws_bytes < ws_need || !lad::aligned(workspace, 16)))
        return set_error(LAD_EWORKSPACE, "kda_prefill_chunked: workspace of %zu bytes (16-byte aligned) required, or NULL",
                         ws_need);
    if (split && static_cast<long long>(B) * H * kSegChunks > 0x7fffffffLL)
        return set_error(LAD_EUNSUPPORTED, "kda_prefill_chunked: B*H too large");
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(kda_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(kda_prefill_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            kPSmemBytes);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(kda_prefill_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            kSSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return set_error(LAD_ECUDA, "kda_prefill_chunked: smem attribute: %s", cudaGetErrorString(attr_err));
    Args a{reinterpret_cast<const uint16_t *>(q), reinterpret_cast<const uint16_t *>(k),
           reinterpret_cast<const uint16_t *>(v), alpha, beta, S, o, B, T, H, scale,
           (flags & LAD_FLAG_L2NORM_QK) ? 1 : 0, f32 ? 1 : 0};
    auto enc = reinterpret_cast<EncodeTiledFn>(lad::tensor_map_encoder_raw());
    if (!enc) return set_error(LAD_ECUDA, "kda_prefill_chunked: cuTensorMapEncodeTiled unavailable");
    Maps maps;
    auto make = [&](CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, int box0) -> int {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(H) * kDk, static_cast<cuuint64_t>(T),
                                    static_cast<cuuint64_t>(B)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(H) * kDk * esize,
                                       static_cast<cuuint64_t>(T) * H * kDk * esize};
        const cuuint32_t box[3] = {static_cast<cuuint32_t>(box0), static_cast<cuuint32_t>(kC), 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        return r == CUDA_SUCCESS ? LAD_OK : set_error(LAD_ECUDA, "kda_prefill_chunked: tensor map failed (%d)", (int)r);
    };
    int rc = make(&maps.q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDk);
    if (rc == LAD_OK) rc = make(&maps.k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDk);
    if (rc == LAD_OK) rc = make(&maps.alpha, alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kDk);
    if (rc == LAD_OK) rc = make(&maps.v, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, split ? kDv : kDvh);
    if (rc != LAD_OK) return rc;
    cudaStream_t st = lad::as_stream(stream);
    if (!split) {
        kda_prefill_kernel<<<static_cast<unsigned>(ctas), kThreads, kSmemBytes, st>>>(a, maps);
        return lad::check_launch("kda_prefill_chunked");
    }
    // split path, segment by segment: every chunk's operands of the segment (prep), then the chain
    const int nch = (T + kC - 1) / kC;
    const int sms = lad::device_sm_count();
    if (sms <= 0) return set_error(LAD_ECUDA, "kda_prefill_chunked: cannot query the SM count");
    for (int c0 = 0; c0 < nch; c0 += kSegChunks) {
        const int nseg = nch - c0 < kSegChunks ? nch - c0 : kSegChunks;
        SplitArgs sa{a.q, a.k, a.v, alpha, beta, S, o, static_cast<uint8_t *>(workspace), B, T, H, c0, nseg,
                     scale, a.l2norm, a.out_f32};
        const long long items = static_cast<long long>(B) * H * nseg;
        const unsigned pg = static_cast<unsigned>(items < sms ? items : sms);
        kda_prefill_prep_kernel<<<pg, kThreads, kPSmemBytes, st>>>(sa, maps);
        rc = lad::check_launch("kda_prefill_chunked");
        if (rc != LAD_OK) return rc;
        kda_prefill_scan_kernel<<<static_cast<unsigned>(ctas), kThreads, kSSmemBytes, st>>>(sa);
        rc = lad::check_launch("kda_prefill_chunked");
        if (rc != LAD_OK) return rc;
    }
    return LAD_OK;
}
