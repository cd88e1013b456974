// Gated MLA latent decode on B200: split-KV over the compressed 576-wide cache, tensor cores
// (tcgen05) for both contractions, TMA-fed, with a log-sum-exp combine and the sigmoid gate.
//
// Sources: "Ling-3.1-flash: a 560B hybrid-attention MoE, counted from its safetensors headers",
// section "How KDA and MLA split the work" (gated MLA is ordinary softmax attention over a
// compressed cache of a 512-dim latent plus a 64-dim RoPE key per token; a sigmoid gate per
// head scales the result); "Ling-3.1-flash and the 7:1 hybrid: how much KV cache does a 560B
// model need at 1M tokens?", section "How big is the cache per token, exactly?" (576 bf16 values
// per token, read in full at every decoding step; 192-wide per-head key, hence 1/sqrt(192)).
//
// For sequence b (L rows c_t) and head h, with the absorbed query q_h (576 wide):
//   s_t = scale <q_h, c_t>,  o_h = sigmoid(g_h) * sum_t softmax(s)_t c_t[0:512].
//
// Work split. Every sequence is cut into tiles of 32 cached rows; the tiles of all sequences,
// concatenated, are divided evenly between one CTA per SM. A CTA's share is a run of
// "segments" (its tiles of one sequence); each segment leaves an unnormalised partial
// (O, running max m, running sum l) in the workspace, and a second kernel merges the partials
// of each sequence by log-sum-exp and applies the gate.
//
// Per tile, two contractions run on the tensor cores (bf16 operands, fp32 accumulation in TMEM):
//   GEMM1  S[h][t]  = q[h][:] . c_t          M = 64 heads, N = 32 tokens, K = 576
//   GEMM2  O^T[d][h] += sum_t c_t[d] P[h][t]  M = 128 latent dims (x4), N = 64 heads, K = 32
// GEMM2 is written transposed so that its M is the 512 latent dimensions and runs at the full
// 128-row rate; its A operand is the same cache tile GEMM1 used as B, read MN-major, so every
// cached byte crosses HBM once. P (bf16) goes through shared memory.
//
// Roles (256 threads): warp 0 issues TMA loads (q once per segment, then a 4-deep ring of
// 36 KiB cache tiles), warp 1 owns TMEM, warps 1 and 2 issue GEMM1, warp 3 GEMM2, warps 4-7 run the online softmax
// (one head per lane, lanes 0-15 of each warp: the M = 64 accumulator occupies rows 16p..16p+15
// of TMEM sub-partition p), rescale O when a head's running max grows by more than 2^8
// (lazily, like FlashAttention-4), and write the segment's partial at its end.
//
// FP8 cache variant (kFp8): rows are 576 E4M3 codes with one fp32 scale for the whole cache. Four
// more warps (8-11) load each tile's codes from global memory straight into registers, two tiles
// ahead (no shared-memory staging: the kernel is bound by shared-memory traffic, not by HBM),
// and write them widened into the same swizzled operand layout and 4-deep ring the TMA fills for
// a bf16 cache; the producer warp then loads only q. The tensor cores run on f16
// operands (kind::f16 takes A and B of one type): an E4M3 pair becomes an f16 pair in one
// conversion (bf16 would take four), every E4M3 value is exact in f16, the query is converted
// bf16 -> f16 in place once per segment (exact within the f16 range; a larger |q| is reported),
// and P is written as f16. The scale folds into the score scale and the combine's normalisation.
//
// Every wait on an mbarrier is bounded (see lad_common.cuh); a wait that runs out records a tag
// in the device error word, raises an abort flag the other roles see, and the CTA drains its
// own copies and MMAs, frees TMEM and returns.
#include <cuda.h>

#include <cstring>
#include <mutex>

#include "sm100_ptx.cuh"

namespace {

using lad::dev::globaltimer_ns;
using lad::dev::kWaitLimitNs;

constexpr int kHq = 64;            // query heads
constexpr int kDl = 512;           // latent (value) width
constexpr int kDr = 64;            // rope width
constexpr int kDrow = kDl + kDr;   // 576 bf16 per cached row
constexpr int kChunk = 64;         // bf16 per 128-byte swizzle row
constexpr int kNChunk = kDrow / kChunk;  // 9
constexpr int kTile = 32;          // cached rows per tile
constexpr int kStages = 4;            // bf16 ring fed by TMA
constexpr int kThreads = 256;
constexpr int kThreadsF8 = 384;       // + 4 converter warps
constexpr int kMaxSplitCtas = 1024;  // one split CTA per SM; the combine tracks at most this many

constexpr int kQChunkBytes = kHq * 128;                 // 8 KiB: 64 heads x 64 dims
constexpr int kQBytes = kNChunk * kQChunkBytes;         // 73,728
constexpr int kTChunkBytes = kTile * 128;               // 4 KiB: 32 rows x 64 dims
constexpr int kStageBytes = kNChunk * kTChunkBytes;     // 36,864
constexpr int kPBytes = kHq * kTile * 2;                // 4 KiB: P[64 heads][32 tokens] bf16

constexpr int kOffQ = 0;
constexpr int kOffStage = kOffQ + kQBytes;                       // 73,728
constexpr int kOffP = kOffStage + kStages * kStageBytes;         // 221,184
constexpr int kOffBar = kOffP + 2 * kPBytes;                     // 229,376
constexpr int kSmemBytes = kOffBar + 1024 + 1024;                // + barriers/scalars + alignment slack

// TMEM columns (fp32): O^T blocks 0..255; S buffer b at 256 + 64 b, holding two partial sums of
// GEMM1 (even and odd K chunks) 32 columns apart, so consecutive MMAs never chain on one
// accumulator.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;
constexpr uint32_t kColS = 256;
constexpr uint32_t kSBufCols = 2 * kTile;

// barrier slots (8 bytes each) inside the kOffBar region
enum Bar : int {
    kBarFull = 0,                 // [kStages]   TMA -> MMA: cache tile landed
    kBarEmpty = kBarFull + kStages,  // [kStages] MMA -> TMA: tile consumed by GEMM2
    kBarSFull = kBarEmpty + kStages,   // [2] GEMM1 done
    kBarSEmpty = kBarSFull + 2,        // [2] softmax has read S
    kBarPFull = kBarSEmpty + 2,        // [2] P written (and O rescaled)
    kBarPEmpty = kBarPFull + 2,        // [2] GEMM2 of the tile that used this P buffer is complete
    kBarWg = kBarPEmpty + 2,           // [2] softmax warps exchanged their rescale decisions
    kBarOFree = kBarWg + 2,            // epilogue has read O
    kBarQFull = kBarOFree + 1,         // q of a segment landed
    kBarQRoped = kBarQFull + 1,        // (RoPE variant) q's RoPE part turned to the query position
    kBarQEmpty = kBarQRoped + 1,       // GEMM1s of a segment done with q
    kBarDrain = kBarQEmpty + 1,        // final MMA drain
    kBarQF16 = kBarDrain + 1,          // (FP8) q converted to f16
    kNumBars = kBarQF16 + 1,
};
constexpr int kOffScalars = kNumBars * 8;  // inside the barrier region: tmem base, abort flag, ...

__device__ int g_mla_error = 0;

// Bounded waits: lad::ptx::wait_bar with this module's device error word (see lad_common.cuh).
// Called by whole warps; the result is warp-uniform, so every lane takes the same path (the issue
// helpers rely on the warp staying converged).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag, int tag) {
    return lad::ptx::wait_bar(bar, parity, abort_flag, &g_mla_error, tag);
}

// The issue helpers (lad::ptx) are executed by a whole, converged warp; `elect.sync` picks one lane
// (the same lowest lane every time) that actually issues. Keeping the warp converged lets the
// descriptors and addresses live in uniform registers, which tcgen05.mma and TMA read directly.
using lad::ptx::e4m3x2_to_f16x2;
using lad::ptx::f32x2_to_f16x2;
using lad::ptx::ex2_approx;
using lad::ptx::fence_async_smem;
using lad::ptx::kLayoutNone;
using lad::ptx::kLayoutSw128;
using lad::ptx::mbar_arrive;
using lad::ptx::mbar_arrive_tx_elect;
using lad::ptx::mbar_init;
using lad::ptx::mbar_try_wait;
using lad::ptx::smem_desc;
using lad::ptx::smem_u32;
using lad::ptx::tc_commit;
using lad::ptx::tc_fence_after;
using lad::ptx::tc_fence_before;
using lad::ptx::tmem_ld32u;
using lad::ptx::tmem_st32u;
using lad::ptx::tmem_wait_ld;
using lad::ptx::tmem_wait_st;

__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    lad::ptx::tc_mma_f16(d, a, b, idesc, acc);
}

// bf16 operands, fp32 accumulator; majors (0 K-major, 1 MN-major)
constexpr uint32_t make_idesc(int M, int N, int a_mn_major, int b_mn_major) {
    return lad::ptx::make_idesc(M, N, lad::ptx::kFmtBf16, a_mn_major, b_mn_major);
}
constexpr uint32_t kIdesc1 = make_idesc(64, kTile, 0, 0);   // S = q . C^T
constexpr uint32_t kIdesc2 = make_idesc(128, kHq, 1, 0);    // O^T += V^T . P^T
// the same with f16 operands (FP8 cache)
constexpr uint32_t kIdesc1F16 = lad::ptx::make_idesc(64, kTile, lad::ptx::kFmtF16, 0, 0);
constexpr uint32_t kIdesc2F16 = lad::ptx::make_idesc(128, kHq, lad::ptx::kFmtF16, 1, 0);

// ------------------------------------------------------------------------------------------
// work split
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ int tiles_of(int len) { return (len + kTile - 1) / kTile; }

__device__ __forceinline__ long long split_point(long long total, int parts, int c) {
    return total * c / parts;
}

// Iterates the segments (runs of tiles of one sequence) of a CTA's tile range [t, t_end).
struct SegIter {
    const int *lens;
    int B;
    int b;             // current sequence
    long long base;    // first global tile of sequence b
    long long t, t_end;

    __device__ bool next(int &seq, int &tile0, int &ntiles) {
        while (t < t_end && b < B) {
            const long long nb = tiles_of(lens[b]);
            if (t < base + nb) {
                const long long end = (t_end < base + nb) ? t_end : base + nb;
                seq = b;
                tile0 = static_cast<int>(t - base);
                ntiles = static_cast<int>(end - t);
                t = end;
                if (t == base + nb) {
                    base += nb;
                    ++b;
                }
                return true;
            }
            base += nb;
            ++b;
        }
        return false;
    }
};

struct Partials {
    float *O;        // [slots][64][512]
    float *m;        // [slots][64]   running max, log2 units of the scaled score
    float *l;        // [slots][64]
    long long *tile_prefix;  // [B + 1]
};

// Paged cache: row t of sequence b is row t % page_size of page block_table[b*bt_stride + t/page_size]
// of a pool of num_pages pages (page_size a multiple of the 32-row tile, so a tile never spans
// two pages). Unused by the contiguous variant.
struct PagedCache {
    const int *block_table;
    int bt_stride;
    int page_size;
    int num_pages;
    int oob_row;  // the pool map's row extent: a tile starting there reads as zeros
};

// RoPE variant: q arrives with its 64-wide RoPE part not yet turned; sequence b's query sits at
// position positions[b]. Pair i (dims i and i + 32, or 2i and 2i + 1 when interleaved) turns by
// positions[b] * inv_freq[i] (inverse frequencies computed on the host).
struct RopeQ {
    const int *positions;
    int interleaved;
    double inv_freq[kDr / 2];
};

// FP8 cache: E4M3 codes, row t of sequence b at base + b * seq_stride + t * 576 (contiguous,
// rows past Lmax read as zeros) or in the page pool at base (paged, rows located as above).
struct Fp8Cache {
    const uint8_t *base;
    long long seq_stride;  // bytes
    int Lmax;
};

// Walks the tiles of a CTA's range in order for the FP8 widening warps: per tile, the address of its
// first row and how many of its rows hold codes to read (0 at or past the length, past Lmax, or in
// a page outside the pool, which is reported). next() is warp-uniform: every lane of a warp calls it.
template <bool kPaged>
struct Fp8Cursor {
    SegIter it;
    const int *seq_lens;
    Fp8Cache f8;
    PagedCache pc;
    int seq, tile0, nt, i, len;
    bool more;
    int pseq, pg0, pg_lane;  // paged: lane j holds block_table[seq][pg0 + j]

    __device__ Fp8Cursor(const SegIter &it_, const int *lens, const Fp8Cache &f, const PagedCache &p)
        : it(it_), seq_lens(lens), f8(f), pc(p), seq(0), tile0(0), nt(0), i(0), len(0), more(true), pseq(-1), pg0(0),
          pg_lane(-1) {}

    __device__ bool next(int lane, const uint8_t *&row0, int &nrows) {
        while (more && i >= nt) {
            more = it.next(seq, tile0, nt);
            i = 0;
            if (more) len = seq_lens[seq];
        }
        if (!more) return false;
        const int t_row = (tile0 + i) * kTile;
        ++i;
        const int lim = kPaged ? len : min(len, f8.Lmax);
        nrows = max(0, min(kTile, lim - t_row));
        if constexpr (kPaged) {
            // 32 block-table entries per load, one per lane
            const int pi = t_row / pc.page_size;
            if (seq != pseq || pi < pg0 || pi >= pg0 + 32) {
                pseq = seq;
                pg0 = pi;
                const int j = pg0 + lane;
                pg_lane = j < pc.bt_stride ? pc.block_table[static_cast<long long>(seq) * pc.bt_stride + j] : -1;
            }
            const int page = __shfl_sync(0xffffffffu, pg_lane, pi - pg0);
            if (page >= 0 && page < pc.num_pages) {
                row0 = f8.base + (static_cast<long long>(page) * pc.page_size + (t_row - pi * pc.page_size)) * kDrow;
            } else {
                if (nrows > 0 && lane == 0) atomicCAS(&g_mla_error, 0, lad::kErrMlaBlockTable);
                row0 = nullptr;
                nrows = 0;
            }
        } else {
            row0 = f8.base + seq * f8.seq_stride + static_cast<long long>(t_row) * kDrow;
        }
        return true;
    }
};

// kPaged: map_cache is 2-D over the page pool ([num_pages * page_size][576]) and each tile's row
// comes from the block table; otherwise it is 3-D ([B][Lmax][576]). kFp8: map_cache is unused and
// the cache is read through f8. cache_group: consecutive sequences that read one cached sequence
// (the query tokens of a multi-token step; 1 otherwise): sequence s reads cached sequence
// s / cache_group of the contiguous map.
template <bool kPaged, bool kRopeQ, bool kFp8>
__global__ void __launch_bounds__(kFp8 ? kThreadsF8 : kThreads, 1)
mla_split_kernel(const __grid_constant__ CUtensorMap map_cache, const __grid_constant__ CUtensorMap map_q,
                 const int *__restrict__ seq_lens, int B, float score_scale_log2, Partials ws, PagedCache pc,
                 const __grid_constant__ RopeQ rq, Fp8Cache f8, int cache_group) {
    constexpr int NSt = kStages;  // depth of the operand ring
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bars = sbase + kOffBar;
    auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
    uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(smem + kOffBar + kOffScalars);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffBar + kOffScalars + 4);
    long long *range = reinterpret_cast<long long *>(smem + kOffBar + kOffScalars + 8);  // [0]=t0 [1]=t1 [2]=b0 [3]=base0
    float *rescale = reinterpret_cast<float *>(smem + kOffBar + kOffScalars + 64);         // [2][64]
    int *any_rescale = reinterpret_cast<int *>(smem + kOffBar + kOffScalars + 64 + 512);   // [2][4]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- the CTA's tile range; warp 2 scans the lengths (and CTA 0 publishes the prefix) ----
    if (warp == 2) {
        long long run = 0;
        for (int b0 = 0; b0 < B; b0 += 32) {
            const int b = b0 + lane;
            long long n = (b < B) ? tiles_of(seq_lens[b]) : 0;
            long long incl = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                long long y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (blockIdx.x == 0 && b < B) ws.tile_prefix[b] = run + incl - n;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (blockIdx.x == 0 && lane == 0) ws.tile_prefix[B] = run;
        if (lane == 0) {
            const long long t0 = split_point(run, gridDim.x, blockIdx.x);
            const long long t1 = split_point(run, gridDim.x, blockIdx.x + 1);
            long long base = 0;
            int b = 0;
            while (b < B) {
                const long long nb = tiles_of(seq_lens[b]);
                if (t0 < base + nb) break;
                base += nb;
                ++b;
            }
            range[0] = t0;
            range[1] = t1;
            range[2] = b;
            range[3] = base;
        }
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            uint32_t count = 1;
            if (i == kBarSEmpty || i == kBarSEmpty + 1 || i == kBarPFull || i == kBarPFull + 1 || i == kBarWg ||
                i == kBarWg + 1 || i == kBarOFree)
                count = 4;  // one arrival per softmax warp
            if (i == kBarSFull || i == kBarSFull + 1 || i == kBarQEmpty)
                count = 2;  // one commit per GEMM1 warp
            if (kFp8 && ((i >= kBarFull && i < kBarFull + NSt) || i == kBarQF16))
                count = 4;  // one arrival per converter warp
            if (i == kBarDrain) count = 3;  // every MMA warp
            mbar_init(bar(i), count);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const long long t0 = range[0], t1 = range[1];
    if (t0 >= t1) return;  // no work for this CTA (uniform exit before TMEM is touched)

    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_base_slot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_slot;

    SegIter it{seq_lens, B, static_cast<int>(range[2]), range[3], t0, t1};

    if (warp == 0) {
        // ================= TMA producer (whole warp, elected lane issues) =================
        {
            int seq, tile0, nt, k = 0;
            uint32_t g = 0;
            bool ok = true;
            // paged: lane j holds block_table[seq][pg0 + j] (-1 past the table's row)
            int pg_seq = -1, pg0 = 0, pg_lane = -1;
            while (ok && it.next(seq, tile0, nt)) {
                if (k > 0 && !wait_bar(bar(kBarQEmpty), (k - 1) & 1, abort_flag, lad::kErrMlaProducer)) {
                    ok = false;
                    break;
                }
                mbar_arrive_tx_elect(bar(kBarQFull), kQBytes);
                for (int c = 0; c < kNChunk; ++c)
                    lad::ptx::tma_load_2d_elect(sbase + kOffQ + c * kQChunkBytes, &map_q, c * kChunk, seq * kHq, bar(kBarQFull));
                // (FP8 cache: the widening warps load the tiles themselves)
                for (int i = 0; i < (kFp8 ? 0 : nt); ++i, ++g) {
                    const uint32_t s = g % NSt;
                    int row = (tile0 + i) * kTile;
                    if constexpr (kPaged) {
                        // warp-uniform: every lane computes the same page index
                        const int pi = row / pc.page_size;
                        if (seq != pg_seq || pi < pg0 || pi >= pg0 + 32) {
                            pg_seq = seq;
                            pg0 = pi;
                            const int j = pg0 + lane;
                            pg_lane = j < pc.bt_stride ? pc.block_table[static_cast<long long>(seq) * pc.bt_stride + j]
                                                       : -1;
                        }
                        const int page = __shfl_sync(0xffffffffu, pg_lane, pi - pg0);
                        if (page >= 0 && page < pc.num_pages) {
                            row = page * pc.page_size + (row - pi * pc.page_size);
                        } else {
                            // a row past the pool: TMA fills the tile with zeros; the call reports it
                            row = pc.oob_row;
                            if (lane == 0) atomicCAS(&g_mla_error, 0, lad::kErrMlaBlockTable);
                        }
                    }
                    if (!wait_bar(bar(kBarEmpty + s), ((g / NSt) & 1) ^ 1, abort_flag, lad::kErrMlaProducer)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_tx_elect(bar(kBarFull + s), kStageBytes);
                    const uint32_t dst = sbase + kOffStage + s * kStageBytes;
                    for (int c = 0; c < kNChunk; ++c) {
                        if constexpr (kPaged)
                            lad::ptx::tma_load_2d_elect(dst + c * kTChunkBytes, &map_cache, c * kChunk, row,
                                                        bar(kBarFull + s));
                        else
                            lad::ptx::tma_load_3d_elect(dst + c * kTChunkBytes, &map_cache, c * kChunk, row,
                                                        seq / cache_group, bar(kBarFull + s));
                    }
                }
                ++k;
            }
            if (!ok) {
                // drain: every load this thread issued completes on its full barrier
                const uint32_t issued = g;
                for (uint32_t j = (issued > NSt ? issued - NSt : 0); j < issued; ++j) {
                    const uint32_t s = j % NSt;
                    const uint64_t tt = globaltimer_ns();
                    while (!mbar_try_wait(bar(kBarFull + s), (j / NSt) & 1) && globaltimer_ns() - tt < kWaitLimitNs) {
                    }
                }
                if (k > 0) {
                    const uint64_t tt = globaltimer_ns();
                    while (!mbar_try_wait(bar(kBarQFull), (k - 1) & 1) && globaltimer_ns() - tt < kWaitLimitNs) {
                    }
                }
            }
        }
    } else if (warp == 1 || warp == 2) {
        // ================= GEMM1 issuers (warps 1 and 2, whole warps, elected lanes issue) =================
        // A single warp issues a small tcgen05.mma only every ~28 cycles, below the tensor pipe's
        // rate for these shapes, so two warps share GEMM1: warp 1 issues the even K chunks into one
        // partial accumulator, warp 2 the odd ones into the other; S_full expects both commits.
        {
            const int mi = warp - 1;
            int seq, tile0, nt, k = 0;
            uint32_t g = 0;
            bool ok = true;
            const uint64_t q_desc0 = smem_desc(sbase + kOffQ, 16, 1024, kLayoutSw128);
            const uint64_t c_desc0 = smem_desc(sbase + kOffStage, 16, 1024, kLayoutSw128);
            while (ok && it.next(seq, tile0, nt)) {
                if (!wait_bar(bar(kFp8 ? kBarQF16 : (kRopeQ ? kBarQRoped : kBarQFull)), k & 1, abort_flag,
                              lad::kErrMlaMma)) {
                    ok = false;
                    break;
                }
                for (int i = 0; i < nt; ++i, ++g) {
                    const uint32_t s = g % NSt;
                    const uint32_t sb = g & 1;
                    if (!wait_bar(bar(kBarFull + s), (g / NSt) & 1, abort_flag, lad::kErrMlaMma) ||
                        !wait_bar(bar(kBarSEmpty + sb), ((g >> 1) & 1) ^ 1, abort_flag, lad::kErrMlaMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t cd = c_desc0 + ((s * kStageBytes) >> 4);
                    const uint32_t dS = tmem + kColS + sb * kSBufCols;
#pragma unroll
                    for (int c = mi; c < kNChunk; c += 2) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc_mma(dS + mi * kTile, q_desc0 + ((c * kQChunkBytes + kk * 32) >> 4),
                                   cd + ((c * kTChunkBytes + kk * 32) >> 4), kFp8 ? kIdesc1F16 : kIdesc1,
                                   (c > 1 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(bar(kBarSFull + sb));
                    if (i == nt - 1) tc_commit(bar(kBarQEmpty));
                }
                ++k;
            }
            // drain every MMA this thread issued before TMEM is released
            tc_commit(bar(kBarDrain));
            const uint64_t tt = globaltimer_ns();
            while (!mbar_try_wait(bar(kBarDrain), 0) && globaltimer_ns() - tt < kWaitLimitNs) {
            }
        }
    } else if (warp == 3) {
        // ================= GEMM2 issuer (warp 3, whole warp, elected lane issues) =================
        // Issued as soon as a tile's P is ready, independently of the next tile's GEMM1, so that the
        // tile's stage goes back to the TMA warp early: the ring is what keeps bytes in flight.
        {
            int seq, tile0, nt, k = 0;
            uint32_t g = 0;
            bool ok = true;
            const uint64_t v_desc0 = smem_desc(sbase + kOffStage, kTChunkBytes, 1024, kLayoutSw128);
            const uint64_t p_desc0 = smem_desc(sbase + kOffP, 128, 512, kLayoutNone);
            while (ok && it.next(seq, tile0, nt)) {
                if constexpr (kRopeQ) {
                    // turn the RoPE part (q dims 512..575: the last 64-dim chunk, one 128-byte
                    // swizzled row per head) to the query position; lane i takes pair i of all heads
                    if (!wait_bar(bar(kBarQFull), k & 1, abort_flag, lad::kErrMlaMma)) {
                        ok = false;
                        break;
                    }
                    double sd, cd;
                    sincos(static_cast<double>(rq.positions[seq]) * rq.inv_freq[lane], &sd, &cd);
                    const float c = static_cast<float>(cd), sn = static_cast<float>(sd);
                    const int ia = rq.interleaved ? 2 * lane : lane;
                    const int ib = rq.interleaved ? 2 * lane + 1 : lane + kDr / 2;
                    uint16_t *qr = reinterpret_cast<uint16_t *>(smem + kOffQ + (kNChunk - 1) * kQChunkBytes);
#pragma unroll 4
                    for (int hh = 0; hh < kHq; ++hh) {
                        // element d of head hh's row: 16-byte chunk (d / 8) xor (hh % 8), slot d % 8
                        uint16_t *row = qr + hh * 64;
                        const int oa = (((ia >> 3) ^ (hh & 7)) << 3) + (ia & 7);
                        const int ob = (((ib >> 3) ^ (hh & 7)) << 3) + (ib & 7);
                        const float x = lad::dev::bf16_to_f32(row[oa]), y = lad::dev::bf16_to_f32(row[ob]);
                        row[oa] = lad::dev::f32_to_bf16(x * c - y * sn);
                        row[ob] = lad::dev::f32_to_bf16(y * c + x * sn);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(kBarQRoped));
                }
                for (int i = 0; i < nt; ++i, ++g) {
                    const uint32_t pb = g & 1;
                    if (!wait_bar(bar(kBarPFull + pb), (g >> 1) & 1, abort_flag, lad::kErrMlaMma)) {
                        ok = false;
                        break;
                    }
                    if (i == 0 && k > 0 && !wait_bar(bar(kBarOFree), (k - 1) & 1, abort_flag, lad::kErrMlaMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t s = g % NSt;
                    // A = V^T: 128 latent dims (two 64-wide chunks, LBO apart) x 16 tokens (two 8-row groups)
                    const uint64_t a0 = v_desc0 + ((s * kStageBytes) >> 4);
                    // B = P: 64 heads (8-row core groups, SBO 512) x 16 tokens (two 8-token core columns, LBO 128)
                    const uint64_t b0 = p_desc0 + ((pb * kPBytes) >> 4);
                    const uint32_t acc0 = i == 0 ? 0u : 1u;
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tc_mma(tmem + kColO + 64 * j, a0 + (((2 * j) * kTChunkBytes + kk * 2048) >> 4),
                                   b0 + ((kk * 256) >> 4), kFp8 ? kIdesc2F16 : kIdesc2, kk == 0 ? acc0 : 1u);
                    }
                    tc_commit(bar(kBarEmpty + s));
                    tc_commit(bar(kBarPEmpty + pb));
                }
                ++k;
            }
            tc_commit(bar(kBarDrain));
            const uint64_t tt = globaltimer_ns();
            while (!mbar_try_wait(bar(kBarDrain), 0) && globaltimer_ns() - tt < kWaitLimitNs) {
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ================= softmax, rescale and epilogue (warps 4..7) =================
        const int p = warp & 3;                 // TMEM sub-partition
        const bool owner = lane < 16;           // this lane owns head 16p + lane
        const int h = 16 * p + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * p) << 16;
        int seq, tile0, nt, k = 0;
        uint32_t g = 0;
        bool ok = true;
        float m = -INFINITY, l = 0.f;
        while (ok && it.next(seq, tile0, nt)) {
            const int len = seq_lens[seq];
            for (int i = 0; i < nt; ++i, ++g) {
                const uint32_t sb = g & 1;
                if (!wait_bar(bar(kBarSFull + sb), (g >> 1) & 1, abort_flag, lad::kErrMlaSoftmax)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t r[kTile], r2[kTile];
                tmem_ld32u(tmem + lane_addr + kColS + sb * kSBufCols, r);
                tmem_ld32u(tmem + lane_addr + kColS + sb * kSBufCols + kTile, r2);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarSEmpty + sb));

                const int tok0 = (tile0 + i) * kTile;
                // the 32 scores of head 16p + (lane % 16) are split over lanes l and l + 16: lane l
                // keeps tokens 0-15 (it loaded the row), lane l + 16 receives tokens 16-31
                const int hi = lane >> 4;
                float xs[kTile / 2];
#pragma unroll
                for (int j = 0; j < kTile / 2; ++j) {
                    const float a = __uint_as_float(r[j]) + __uint_as_float(r2[j]);
                    const float b = __uint_as_float(r[16 + j]) + __uint_as_float(r2[16 + j]);
                    const float from_low = __shfl_sync(0xffffffffu, b, lane & 15);
                    xs[j] = hi ? from_low : a;
                }
                const int mytok0 = tok0 + 16 * hi;
                if (tok0 + kTile > len) {
#pragma unroll
                    for (int j = 0; j < kTile / 2; ++j)
                        if (mytok0 + j >= len) xs[j] = -INFINITY;
                }
                if (!kFp8 && tok0 + kTile > len) {  // (the FP8 converter already wrote those rows as zeros)
                    // Rows past the length get weight 0, but 0 * (NaN or Inf) would still reach O:
                    // zero their latent part in the stage (GEMM1 is done with it, GEMM2 waits for
                    // P_full, which follows the proxy fence below).
                    const int valid = len - tok0;
                    uint8_t *stage = smem + kOffStage + (g % NSt) * kStageBytes;
                    for (int idx = threadIdx.x - 128; idx < (kTile - valid) * 64; idx += 128) {
                        const int rr = valid + (idx >> 6);
                        const int c = (idx >> 3) & 7;
                        *reinterpret_cast<uint4 *>(stage + c * kTChunkBytes + rr * 128 + (idx & 7) * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                // scores stay unscaled; the scale (with log2 e) is folded into the exponent below
                float t8[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) t8[j] = fmaxf(xs[j], xs[j + 8]);
#pragma unroll
                for (int j = 0; j < 4; ++j) t8[j] = fmaxf(t8[j], t8[j + 4]);
                float tmax = fmaxf(fmaxf(t8[0], t8[2]), fmaxf(t8[1], t8[3]));
                tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
                tmax *= score_scale_log2;
                if (i == 0) {
                    m = -INFINITY;
                    l = 0.f;
                }
                float f = 1.f;
                bool need = false;
                if (m == -INFINITY) {
                    m = tmax;
                    f = 0.f;
                } else if (tmax > m + 8.f) {
                    f = ex2_approx(m - tmax);
                    m = tmax;
                    need = true;
                }
                uint32_t pk[kTile / 4];
                float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < kTile / 2; j += 2) {
                    const float p0 = ex2_approx(fmaf(xs[j], score_scale_log2, -m));
                    const float p1 = ex2_approx(fmaf(xs[j + 1], score_scale_log2, -m));
                    ps[(j >> 1) & 3] += p0 + p1;  // the denominator keeps fp32 probabilities
                    pk[j / 2] = kFp8 ? f32x2_to_f16x2(p0, p1) : lad::dev::f32x2_to_bf16x2(p0, p1);
                }
                float psum = (ps[0] + ps[1]) + (ps[2] + ps[3]);
                psum += __shfl_xor_sync(0xffffffffu, psum, 16);
                l = l * f + psum;

                const uint32_t pb = g & 1;
                if (!wait_bar(bar(kBarPEmpty + pb), ((g >> 1) & 1) ^ 1, abort_flag, lad::kErrMlaSoftmax)) {
                    ok = false;
                    break;
                }
                const uint32_t rb = g & 1;
                {
                    // P[h][t], K-major without swizzle: 8x8 core matrices of 128 bytes; head group
                    // h/8 at 512 B, token group t/8 at 128 B, row h%8 at 16 B. This lane's 16 tokens
                    // are token groups 2*hi and 2*hi + 1.
                    const int hh = 16 * p + (lane & 15);
                    uint8_t *prow = smem + kOffP + pb * kPBytes + (hh >> 3) * 512 + (hh & 7) * 16 + 2 * hi * 128;
                    *reinterpret_cast<uint4 *>(prow) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4 *>(prow + 128) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    if (owner) rescale[rb * 64 + h] = f;
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                const int any = __any_sync(0xffffffffu, owner && need);
                if (lane == 0) any_rescale[rb * 4 + p] = any;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarWg + rb));
                if (!wait_bar(bar(kBarWg + rb), (g >> 1) & 1, abort_flag, lad::kErrMlaSoftmax)) {
                    ok = false;
                    break;
                }
                const bool do_rescale = (any_rescale[rb * 4 + 0] | any_rescale[rb * 4 + 1] |
                                         any_rescale[rb * 4 + 2] | any_rescale[rb * 4 + 3]) != 0;
                if (do_rescale) {
                    // GEMM2 of the previous tile (same segment, since i > 0) must be complete
                    const uint32_t gp = g - 1;
                    if (!wait_bar(bar(kBarPEmpty + (gp & 1)), (gp >> 1) & 1, abort_flag, lad::kErrMlaSoftmax)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int j = 0; j < 4; ++j) {
#pragma unroll 1
                        for (int half = 0; half < 2; ++half) {
                            uint32_t o[32];
                            const uint32_t ta = tmem + lane_addr + kColO + 64 * j + 32 * half;
                            tmem_ld32u(ta, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                o[c] = __float_as_uint(__uint_as_float(o[c]) * rescale[rb * 64 + 32 * half + c]);
                            tmem_st32u(ta, o);
                        }
                    }
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarPFull + pb));

                if (i == nt - 1) {
                    // ---- segment epilogue: O^T (unnormalised), m and l to the workspace ----
                    if (!wait_bar(bar(kBarPEmpty + (g & 1)), (g >> 1) & 1, abort_flag, lad::kErrMlaEpilogue)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const long long slot = static_cast<long long>(blockIdx.x) + seq;
                    float *Od = ws.O + slot * (kHq * kDl);
#pragma unroll 1
                    for (int j = 0; j < 4; ++j) {
                        const int d = 128 * j + 32 * p + lane;
#pragma unroll 1
                        for (int half = 0; half < 2; ++half) {
                            uint32_t o[32];
                            tmem_ld32u(tmem + lane_addr + kColO + 64 * j + 32 * half, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int c = 0; c < 32; ++c) Od[(32 * half + c) * kDl + d] = __uint_as_float(o[c]);
                        }
                    }
                    if (owner) {
                        ws.m[slot * kHq + h] = m;
                        ws.l[slot * kHq + h] = l;
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(kBarOFree));
                }
            }
            ++k;
        }
        (void)ok;
    } else if constexpr (kFp8) {
        // ================= FP8 widening (warps 8..11) =================
        // Per segment, q (bf16, turned in the RoPE variant) becomes f16 in place. Per tile, thread
        // (r, jj) holds codes 16jj..16jj+15 of row r of each of the 9 64-wide chunks (9 x 16 bytes),
        // loaded two tiles ahead into one of two register sets, and writes them widened as two
        // 16-byte pieces of the swizzled f16 row. Rows at or past the length (or Lmax, or in a page
        // outside the pool) are not loaded and become zeros.
        const int ct = static_cast<int>(threadIdx.x) - 256;
        const int r = ct >> 2, jj = ct & 3;
        const uint32_t o0 = static_cast<uint32_t>(r * 128 + (((2 * jj) ^ (r & 7)) << 4));
        const uint32_t o1 = static_cast<uint32_t>(r * 128 + (((2 * jj + 1) ^ (r & 7)) << 4));
        // The load cursor runs two tiles ahead of the conversion (two register sets).
        Fp8Cursor<kPaged> cl(it, seq_lens, f8, pc);
        auto load_next = [&](uint4 (&buf)[kNChunk]) {
            const uint8_t *p = nullptr;
            int n = 0;
            if (!cl.next(lane, p, n)) n = 0;
            const uint8_t *src = r < n ? p + r * kDrow + jj * 16 : nullptr;
#pragma unroll
            for (int c = 0; c < kNChunk; ++c) {
                if (src) {
                    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(buf[c].x), "=r"(buf[c].y), "=r"(buf[c].z), "=r"(buf[c].w)
                                 : "l"(src + c * kChunk));
                } else {
                    buf[c] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
        };
        auto widen = [&](const uint4 (&buf)[kNChunk], uint8_t *dst) {
#pragma unroll
            for (int c = 0; c < kNChunk; ++c) {
                const uint4 in = buf[c];
                *reinterpret_cast<uint4 *>(dst + c * kTChunkBytes + o0) =
                    make_uint4(e4m3x2_to_f16x2(in.x), e4m3x2_to_f16x2(in.x >> 16), e4m3x2_to_f16x2(in.y),
                               e4m3x2_to_f16x2(in.y >> 16));
                *reinterpret_cast<uint4 *>(dst + c * kTChunkBytes + o1) =
                    make_uint4(e4m3x2_to_f16x2(in.z), e4m3x2_to_f16x2(in.z >> 16), e4m3x2_to_f16x2(in.w),
                               e4m3x2_to_f16x2(in.w >> 16));
            }
        };
        uint4 bufA[kNChunk], bufB[kNChunk];
        load_next(bufA);
        load_next(bufB);
        int seq, tile0, nt, k = 0;
        uint32_t g = 0;
        bool ok = true;
        while (ok && it.next(seq, tile0, nt)) {
            if (!wait_bar(bar(kRopeQ ? kBarQRoped : kBarQFull), k & 1, abort_flag, lad::kErrMlaConvert)) {
                ok = false;
                break;
            }
            {
                uint4 *qv = reinterpret_cast<uint4 *>(smem + kOffQ);
                bool over = false;
#pragma unroll 2
                for (int i = ct; i < kQBytes / 16; i += 128) {
                    const uint4 w = qv[i];
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                    uint32_t hs[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float lo = __uint_as_float(ws[u] << 16), hi = __uint_as_float(ws[u] & 0xffff0000u);
                        over |= fabsf(lo) > 65504.f || fabsf(hi) > 65504.f;
                        hs[u] = f32x2_to_f16x2(lo, hi);
                    }
                    qv[i] = make_uint4(hs[0], hs[1], hs[2], hs[3]);
                }
                if (__any_sync(0xffffffffu, over) && lane == 0) atomicCAS(&g_mla_error, 0, lad::kErrMlaQRange);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarQF16));
            }
            ++k;
            for (int i = 0; i < nt; ++i, ++g) {
                const uint32_t s = g % NSt;
                if (!wait_bar(bar(kBarEmpty + s), ((g / NSt) & 1) ^ 1, abort_flag, lad::kErrMlaConvert)) {
                    ok = false;
                    break;
                }
                uint8_t *dst = smem + kOffStage + s * kStageBytes;
                if (g & 1) {
                    widen(bufB, dst);
                    load_next(bufB);
                } else {
                    widen(bufA, dst);
                    load_next(bufA);
                }
                fence_async_smem();  // the tensor core (async proxy) reads what these stores wrote
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarFull + s));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

// Merges the partials of each sequence by log-sum-exp, normalises and applies the gate.
// Grid (B, 64 heads), 128 threads, 4 latent dims per thread.
template <bool kOutF32>
__global__ void __launch_bounds__(128)
mla_combine_kernel(const int *__restrict__ seq_lens, int B, int G, const float *__restrict__ gate,
                   Partials ws, void *__restrict__ out, float *__restrict__ lse_out, float value_scale) {
    const int b = blockIdx.x, h = blockIdx.y;
    const int d = 4 * threadIdx.x;
    __shared__ int s_c[2];
    const long long total = ws.tile_prefix[B];
    const long long lo = ws.tile_prefix[b], hi = ws.tile_prefix[b + 1];
    if (threadIdx.x == 0) {
        // CTAs whose tile range [split(c), split(c+1)) meets [lo, hi): start from the estimate
        // lo*G/total and correct it (split points are floor(total*c/G)).
        int c0 = 0, c1 = -1;
        if (hi > lo) {
            c0 = static_cast<int>(lo * G / total);
            while (c0 > 0 && split_point(total, G, c0) > lo) --c0;
            while (split_point(total, G, c0 + 1) <= lo) ++c0;
            c1 = static_cast<int>((hi - 1) * G / total);
            while (c1 > 0 && split_point(total, G, c1) > hi - 1) --c1;
            while (split_point(total, G, c1 + 1) <= hi - 1) ++c1;
        }
        s_c[0] = c0;
        s_c[1] = c1;
    }
    __syncthreads();
    const int c0 = s_c[0], c1 = s_c[1];
    // Per covering CTA its partial's weight, in shared memory: 0 for a CTA that owns no tiles (with
    // fewer tiles than CTAs) and so wrote no partial. Then every thread runs over the partials with
    // independent loads.
    __shared__ float s_w[kMaxSplitCtas];
    __shared__ float s_red[4];
    const int nc = c1 - c0 + 1;
    float mx = -INFINITY;
    for (int i = static_cast<int>(threadIdx.x); i < nc; i += blockDim.x) {
        const int c = c0 + i;
        const bool valid = split_point(total, G, c) < split_point(total, G, c + 1);
        const float mc = valid ? ws.m[(static_cast<long long>(c) + b) * kHq + h] : -INFINITY;
        s_w[i] = mc;
        mx = fmaxf(mx, mc);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = mx;
    __syncthreads();
    const float M = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
    float ls = 0.f;
    for (int i = static_cast<int>(threadIdx.x); i < nc; i += blockDim.x) {
        const float mc = s_w[i];
        const float w = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
        s_w[i] = w;
        if (w != 0.f) ls = fmaf(w, ws.l[(static_cast<long long>(c0 + i) + b) * kHq + h], ls);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
    __syncthreads();  // s_red is reused below; s_w is complete
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ls;
    __syncthreads();
    const float Lsum = (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float *Ob = ws.O + (static_cast<long long>(c0 + b) * kHq + h) * kDl + d;
    const long long slot_stride = static_cast<long long>(kHq) * kDl;
#pragma unroll 4
    for (int i = 0; i < nc; ++i) {
        const float w = s_w[i];
        if (w != 0.f) {
            const float4 v = *reinterpret_cast<const float4 *>(Ob + i * slot_stride);
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
        }
    }
    float sc = (Lsum > 0.f) ? value_scale / Lsum : 0.f;
    if (gate) sc *= 1.f / (1.f + expf(-gate[b * kHq + h]));
    acc.x *= sc;
    acc.y *= sc;
    acc.z *= sc;
    acc.w *= sc;
    const long long o_off = (static_cast<long long>(b) * kHq + h) * kDl + d;
    if constexpr (kOutF32) {
        *reinterpret_cast<float4 *>(static_cast<float *>(out) + o_off) = acc;
    } else {
        uint2 pk;
        pk.x = lad::dev::f32x2_to_bf16x2(acc.x, acc.y);
        pk.y = lad::dev::f32x2_to_bf16x2(acc.z, acc.w);
        *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(out) + o_off) = pk;
    }
    if (lse_out && threadIdx.x == 0)
        lse_out[b * kHq + h] = (Lsum > 0.f) ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WsLayout {
    size_t off_O, off_m, off_l, off_prefix, total;
};

WsLayout ws_layout(int B, int G) {
    const size_t slots = static_cast<size_t>(G) + static_cast<size_t>(B);
    WsLayout w{};
    w.off_O = 0;
    w.off_m = align_up(w.off_O + slots * kHq * kDl * sizeof(float), 256);
    w.off_l = align_up(w.off_m + slots * kHq * sizeof(float), 256);
    w.off_prefix = align_up(w.off_l + slots * kHq * sizeof(float), 256);
    w.total = align_up(w.off_prefix + (static_cast<size_t>(B) + 1) * sizeof(long long), 256);
    return w;
}

}  // namespace

namespace lad {
int take_device_error_mla(cudaStream_t s, int *code) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_mla_error, sizeof v, 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return set_error(LAD_ECUDA, "lad_device_error: %s", cudaGetErrorString(e));
    if (v) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_mla_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return set_error(LAD_ECUDA, "lad_device_error: %s", cudaGetErrorString(e));
    }
    *code = v;
    return LAD_OK;
}
}  // namespace lad

namespace {

// Per-device one-time setup of the split kernels' shared-memory limit.
int set_smem_attributes(const char *name) {
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return lad::set_error(LAD_ECUDA, "%s: %s", name, cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return lad::set_error(LAD_EUNSUPPORTED, "%s: device %d", name, dev);
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
        const void *kernels[] = {
            reinterpret_cast<const void *>(mla_split_kernel<false, false, false>),
            reinterpret_cast<const void *>(mla_split_kernel<true, false, false>),
            reinterpret_cast<const void *>(mla_split_kernel<true, true, false>),
            reinterpret_cast<const void *>(mla_split_kernel<false, false, true>),
            reinterpret_cast<const void *>(mla_split_kernel<true, false, true>),
            reinterpret_cast<const void *>(mla_split_kernel<true, true, true>),
        };
        for (const void *k : kernels) {
            e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            if (e != cudaSuccess) break;
        }
        if (e != cudaSuccess)
            return lad::set_error(LAD_ECUDA, "%s: smem attribute: %s", name, cudaGetErrorString(e));
        done[dev] = true;
    }
    return LAD_OK;
}

// Checks shared by every entry point (B == 0 is handled by the caller after these).
int check_common(const char *name, int B, int Hq, int d_latent, int d_rope, unsigned flags, float scale) {
    using lad::set_error;
    if (B < 0) return set_error(LAD_EINVAL, "%s: negative B", name);
    if (Hq != kHq || d_latent != kDl || d_rope != kDr)
        return set_error(LAD_EUNSUPPORTED, "%s: Hq = 64, d_latent = 512, d_rope = 64 only", name);
    if (flags & ~LAD_FLAG_OUT_FP32) return set_error(LAD_EINVAL, "%s: unknown flags 0x%x", name, flags);
    if (!(scale > 0.f) || scale == INFINITY) return set_error(LAD_EINVAL, "%s: scale must be positive", name);
    return LAD_OK;
}

int check_pointers(const char *name, const void *q, const void *cache, const int *seq_lens, const void *o,
                   unsigned flags) {
    using lad::set_error;
    if (!q || !cache || !seq_lens || !o) return set_error(LAD_EINVAL, "%s: null pointer", name);
    if (!lad::aligned(q, 16) || !lad::aligned(cache, 16))
        return set_error(LAD_EUNSUPPORTED, "%s: q and the cache must be 16-byte aligned", name);
    if (!lad::aligned(o, (flags & LAD_FLAG_OUT_FP32) ? 16 : 8))
        return set_error(LAD_EUNSUPPORTED, "%s: o misaligned", name);
    return LAD_OK;
}

// Tiles of 32 rows x 64 columns (one 128-byte swizzle row each), 128-byte swizzle.
int encode_cache_map(const char *name, CUtensorMap *map, const lad_bf16 *base, int rank, const cuuint64_t *dims,
                     const cuuint64_t *strides) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return lad::set_error(LAD_ECUDA, "%s: cuTensorMapEncodeTiled unavailable", name);
    const cuuint32_t box[3] = {kChunk, kTile, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<lad_bf16 *>(base), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return lad::set_error(LAD_ECUDA, "%s: cache tensor map failed (%d)", name, (int)r);
    return LAD_OK;
}

// Contiguous cache [B][Lmax][576] with a sequence stride (elements).
int encode_contiguous(const char *name, CUtensorMap *map, const lad_bf16 *cache, int B, int Lmax,
                      long long seq_stride) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDrow), static_cast<cuuint64_t>(Lmax),
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDrow) * 2, static_cast<cuuint64_t>(seq_stride) * 2};
    return encode_cache_map(name, map, cache, 3, dims, strides);
}

// Everything after the argument checks: the q map, the split kernel and the combine. f8 non-null:
// the cache is FP8 (map_cache unused), every element worth kv_scale times its code.
int run_mla(const char *name, const CUtensorMap &map_cache, bool paged, const PagedCache &pc, const RopeQ *rope,
            const lad_bf16 *q, const int *seq_lens, const float *gate_logits, void *o, float *lse_out, int B,
            float scale, unsigned flags, uint8_t *ws, const WsLayout &wl, int G, void *stream,
            const Fp8Cache *f8 = nullptr, float kv_scale = 1.f, int cache_group = 1) {
    using lad::set_error;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return set_error(LAD_ECUDA, "%s: cuTensorMapEncodeTiled unavailable", name);
    CUtensorMap map_q;
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDrow), static_cast<cuuint64_t>(B) * kHq};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDrow) * 2};
        const cuuint32_t box[2] = {kChunk, kHq};
        const cuuint32_t estr[2] = {1, 1};
        CUresult r = enc(&map_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<lad_bf16 *>(q), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return set_error(LAD_ECUDA, "%s: q tensor map failed (%d)", name, (int)r);
    }
    int rc = set_smem_attributes(name);
    if (rc != LAD_OK) return rc;
    // Every slot the combine reads is written earlier in the same call (partials by their CTA's
    // epilogue, the tile prefix by CTA 0), so nothing left over from a previous call is read.
    Partials parts{reinterpret_cast<float *>(ws + wl.off_O), reinterpret_cast<float *>(ws + wl.off_m),
                   reinterpret_cast<float *>(ws + wl.off_l), reinterpret_cast<long long *>(ws + wl.off_prefix)};
    cudaStream_t s = lad::as_stream(stream);
    const float score_scale_log2 = scale * kv_scale * 1.4426950408889634f;
    const RopeQ none{};
    const RopeQ &rq = rope ? *rope : none;
    const Fp8Cache fc = f8 ? *f8 : Fp8Cache{};
    if (f8) {
        if (rope)
            mla_split_kernel<true, true, true><<<G, kThreadsF8, kSmemBytes, s>>>(map_cache, map_q, seq_lens, B,
                                                                                 score_scale_log2, parts, pc, rq, fc, cache_group);
        else if (paged)
            mla_split_kernel<true, false, true><<<G, kThreadsF8, kSmemBytes, s>>>(map_cache, map_q, seq_lens, B,
                                                                                  score_scale_log2, parts, pc, rq, fc, cache_group);
        else
            mla_split_kernel<false, false, true><<<G, kThreadsF8, kSmemBytes, s>>>(map_cache, map_q, seq_lens, B,
                                                                                   score_scale_log2, parts, pc, rq, fc, cache_group);
    } else if (rope) {
        mla_split_kernel<true, true, false><<<G, kThreads, kSmemBytes, s>>>(map_cache, map_q, seq_lens, B,
                                                                            score_scale_log2, parts, pc, rq, fc, cache_group);
    } else if (paged) {
        mla_split_kernel<true, false, false><<<G, kThreads, kSmemBytes, s>>>(map_cache, map_q, seq_lens, B,
                                                                             score_scale_log2, parts, pc, rq, fc, cache_group);
    } else {
        mla_split_kernel<false, false, false><<<G, kThreads, kSmemBytes, s>>>(map_cache, map_q, seq_lens, B,
                                                                              score_scale_log2, parts, pc, rq, fc, cache_group);
    }
    rc = lad::check_launch(name);
    if (rc != LAD_OK) return rc;
    const dim3 cgrid(static_cast<unsigned>(B), kHq);
    if (flags & LAD_FLAG_OUT_FP32)
        mla_combine_kernel<true><<<cgrid, 128, 0, s>>>(seq_lens, B, G, gate_logits, parts, o, lse_out, kv_scale);
    else
        mla_combine_kernel<false><<<cgrid, 128, 0, s>>>(seq_lens, B, G, gate_logits, parts, o, lse_out, kv_scale);
    return lad::check_launch(name);
}

int sm_count_checked(const char *name, int *G) {
    *G = lad::device_sm_count();
    if (*G <= 0) return lad::set_error(LAD_ECUDA, "%s: cannot query the SM count", name);
    if (*G > kMaxSplitCtas) return lad::set_error(LAD_EUNSUPPORTED, "%s: more than %d SMs", name, kMaxSplitCtas);
    return LAD_OK;
}

}  // namespace

extern "C" size_t mla_latent_decode_workspace_size(int B, int Hq, int d_latent, int num_sms) {
    if (B < 0 || Hq != kHq || d_latent != kDl) return 0;
    const int G = num_sms > 0 ? num_sms : lad::device_sm_count();
    if (G <= 0) return 0;
    return ws_layout(B, G).total;
}

extern "C" int mla_latent_decode(const lad_bf16 *q, const lad_bf16 *cache, long long cache_seq_stride,
                                 const int *seq_lens, const float *gate_logits, void *o, float *lse_out, int B, int Hq,
                                 int d_latent, int d_rope, int Lmax, float scale, unsigned flags, void *workspace,
                                 size_t ws_bytes, void *stream) {
    using lad::set_error;
    const char *name = "mla_latent_decode";
    int rc = check_common(name, B, Hq, d_latent, d_rope, flags, scale);
    if (rc != LAD_OK) return rc;
    if (Lmax < 0) return set_error(LAD_EINVAL, "%s: negative Lmax", name);
    if (B == 0) return LAD_OK;
    rc = check_pointers(name, q, cache, seq_lens, o, flags);
    if (rc != LAD_OK) return rc;
    if (Lmax == 0) Lmax = 1;  // every length is then 0; the tensor map still needs a non-empty extent
    if (cache_seq_stride < static_cast<long long>(Lmax) * kDrow || cache_seq_stride % 8 != 0)
        return set_error(LAD_EINVAL, "%s: cache_seq_stride must be >= Lmax*576 and a multiple of 8", name);
    int G = 0;
    rc = sm_count_checked(name, &G);
    if (rc != LAD_OK) return rc;
    const WsLayout wl = ws_layout(B, G);
    if (!workspace || ws_bytes < wl.total || !lad::aligned(workspace, 256))
        return set_error(LAD_EWORKSPACE, "%s: workspace of %zu bytes (256-aligned) required", name, wl.total);
    CUtensorMap map_cache;
    rc = encode_contiguous(name, &map_cache, cache, B, Lmax, cache_seq_stride);
    if (rc != LAD_OK) return rc;
    return run_mla(name, map_cache, false, PagedCache{}, nullptr, q, seq_lens, gate_logits, o, lse_out, B, scale,
                   flags, static_cast<uint8_t *>(workspace), wl, G, stream);
}

namespace {
int run_paged(const char *name, const lad_bf16 *q, const void *kv_pages, int num_pages, int page_size,
              const int *block_table, int block_table_stride, const int *seq_lens, const float *gate_logits, void *o,
              float *lse_out, int B, int Hq, int d_latent, int d_rope, float scale, unsigned flags,
              unsigned extra_flags, const RopeQ *rope, void *workspace, size_t ws_bytes, void *stream,
              bool fp8 = false, float kv_scale = 1.f) {
    using lad::set_error;
    int rc = check_common(name, B, Hq, d_latent, d_rope, flags & ~extra_flags, scale);
    if (rc != LAD_OK) return rc;
    if (num_pages < 0 || block_table_stride < 0) return set_error(LAD_EINVAL, "%s: negative size", name);
    if (page_size <= 0 || page_size % kTile != 0)
        return set_error(LAD_EUNSUPPORTED, "%s: page_size must be a positive multiple of %d", name, kTile);
    if (static_cast<long long>(num_pages) * page_size > 0x7fffffffLL - page_size)
        return set_error(LAD_EUNSUPPORTED, "%s: the pool holds more than 2^31 rows", name);
    if (B == 0) return LAD_OK;
    rc = check_pointers(name, q, kv_pages, seq_lens, o, flags);
    if (rc != LAD_OK) return rc;
    if (!block_table) return set_error(LAD_EINVAL, "%s: null block table", name);
    int G = 0;
    rc = sm_count_checked(name, &G);
    if (rc != LAD_OK) return rc;
    const WsLayout wl = ws_layout(B, G);
    if (!workspace || ws_bytes < wl.total || !lad::aligned(workspace, 256))
        return set_error(LAD_EWORKSPACE, "%s: workspace of %zu bytes (256-aligned) required", name, wl.total);
    CUtensorMap map_cache;
    std::memset(&map_cache, 0, sizeof map_cache);
    // an empty pool still gets a one-row extent; every tile then reads as zeros
    const int rows = num_pages > 0 ? num_pages * page_size : 1;
    if (!fp8) {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDrow), static_cast<cuuint64_t>(rows)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDrow) * 2};
        rc = encode_cache_map(name, &map_cache, static_cast<const lad_bf16 *>(kv_pages), 2, dims, strides);
        if (rc != LAD_OK) return rc;
    }
    const PagedCache pc{block_table, block_table_stride, page_size, num_pages, rows};
    const Fp8Cache f8{static_cast<const uint8_t *>(kv_pages), 0, 0};
    return run_mla(name, map_cache, true, pc, rope, q, seq_lens, gate_logits, o, lse_out, B, scale,
                   flags & ~extra_flags, static_cast<uint8_t *>(workspace), wl, G, stream, fp8 ? &f8 : nullptr,
                   kv_scale);
}
}  // namespace

extern "C" int mla_latent_decode_paged(const lad_bf16 *q, const lad_bf16 *kv_pages, int num_pages, int page_size,
                                       const int *block_table, int block_table_stride, const int *seq_lens,
                                       const float *gate_logits, void *o, float *lse_out, int B, int Hq, int d_latent,
                                       int d_rope, float scale, unsigned flags, void *workspace, size_t ws_bytes,
                                       void *stream) {
    return run_paged("mla_latent_decode_paged", q, kv_pages, num_pages, page_size, block_table, block_table_stride,
                     seq_lens, gate_logits, o, lse_out, B, Hq, d_latent, d_rope, scale, flags, 0u, nullptr, workspace,
                     ws_bytes, stream);
}

extern "C" int mla_latent_decode_paged_rope(const lad_bf16 *q, const int *positions, float rope_theta,
                                            const lad_bf16 *kv_pages, int num_pages, int page_size,
                                            const int *block_table, int block_table_stride, const int *seq_lens,
                                            const float *gate_logits, void *o, float *lse_out, int B, int Hq,
                                            int d_latent, int d_rope, float scale, unsigned flags, void *workspace,
                                            size_t ws_bytes, void *stream) {
    const char *name = "mla_latent_decode_paged_rope";
    if (B > 0 && !positions) return lad::set_error(LAD_EINVAL, "%s: null positions", name);
    if (!(rope_theta > 1.f) || rope_theta == INFINITY)
        return lad::set_error(LAD_EINVAL, "%s: rope_theta must be > 1", name);
    RopeQ rq{};
    rq.positions = positions;
    rq.interleaved = (flags & LAD_FLAG_ROPE_INTERLEAVED) ? 1 : 0;
    if (d_rope == kDr) lad::rope_inverse_frequencies(static_cast<double>(rope_theta), kDr, rq.inv_freq);
    return run_paged(name, q, kv_pages, num_pages, page_size, block_table, block_table_stride, seq_lens, gate_logits,
                     o, lse_out, B, Hq, d_latent, d_rope, scale, flags, LAD_FLAG_ROPE_INTERLEAVED, &rq, workspace,
                     ws_bytes, stream);
}

// ------------------------------------------------------------------------------------------
// Multi-token step (the T query tokens of a speculative-decoding verify): the last T of a
// sequence's L cached rows are the T tokens' own rows, and token j attends rows 0 .. L - T + j.
// Every token is a sequence of its own to the split kernel (cache_group = T: T consecutive
// ones read one cached sequence), with its length written by a small kernel into the workspace.
// ------------------------------------------------------------------------------------------
namespace {
__global__ void mla_multi_lens_kernel(const int *__restrict__ seq_lens, int B, int T, int *__restrict__ vlens) {
    const int v = blockIdx.x * blockDim.x + threadIdx.x;
    if (v < B * T) {
        const int b = v / T, j = v - b * T;
        const int L = seq_lens[b] - (T - 1 - j);
        vlens[v] = L > 0 ? L : 0;
    }
}

size_t multi_ws_bytes(int BT, int G) {
    return ws_layout(BT, G).total + align_up(static_cast<size_t>(BT) * sizeof(int), 256);
}
}  // namespace

extern "C" size_t mla_latent_decode_multi_workspace_size(int B, int T, int Hq, int d_latent, int num_sms) {
    if (B < 0 || T < 1 || Hq != kHq || d_latent != kDl || static_cast<long long>(B) * T > 0x7fffffffLL) return 0;
    const int G = num_sms > 0 ? num_sms : lad::device_sm_count();
    if (G <= 0) return 0;
    return multi_ws_bytes(B * T, G);
}

extern "C" int mla_latent_decode_multi(const lad_bf16 *q, const lad_bf16 *cache, long long cache_seq_stride,
                                       const int *seq_lens, const float *gate_logits, void *o, float *lse_out, int B,
                                       int T, int Hq, int d_latent, int d_rope, int Lmax, float scale, unsigned flags,
                                       void *workspace, size_t ws_bytes, void *stream) {
    using lad::set_error;
    const char *name = "mla_latent_decode_multi";
    int rc = check_common(name, B, Hq, d_latent, d_rope, flags, scale);
    if (rc != LAD_OK) return rc;
    if (T < 1) return set_error(LAD_EINVAL, "%s: T must be at least 1", name);
    if (static_cast<long long>(B) * T > 0x7fffffffLL) return set_error(LAD_EUNSUPPORTED, "%s: B*T too large", name);
    if (Lmax < 0) return set_error(LAD_EINVAL, "%s: negative Lmax", name);
    if (B == 0) return LAD_OK;
    rc = check_pointers(name, q, cache, seq_lens, o, flags);
    if (rc != LAD_OK) return rc;
    if (Lmax == 0) Lmax = 1;
    if (cache_seq_stride < static_cast<long long>(Lmax) * kDrow || cache_seq_stride % 8 != 0)
        return set_error(LAD_EINVAL, "%s: cache_seq_stride must be >= Lmax*576 and a multiple of 8", name);
    int G = 0;
    rc = sm_count_checked(name, &G);
    if (rc != LAD_OK) return rc;
    const int BT = B * T;
    const WsLayout wl = ws_layout(BT, G);
    if (!workspace || ws_bytes < multi_ws_bytes(BT, G) || !lad::aligned(workspace, 256))
        return set_error(LAD_EWORKSPACE, "%s: workspace of %zu bytes (256-aligned) required", name,
                         multi_ws_bytes(BT, G));
    int *vlens = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + wl.total);
    cudaStream_t s = lad::as_stream(stream);
    mla_multi_lens_kernel<<<(BT + 255) / 256, 256, 0, s>>>(seq_lens, B, T, vlens);
    rc = lad::check_launch(name);
    if (rc != LAD_OK) return rc;
    CUtensorMap map_cache;
    rc = encode_contiguous(name, &map_cache, cache, B, Lmax, cache_seq_stride);
    if (rc != LAD_OK) return rc;
    return run_mla(name, map_cache, false, PagedCache{}, nullptr, q, vlens, gate_logits, o, lse_out, BT, scale, flags,
                   static_cast<uint8_t *>(workspace), wl, G, stream, nullptr, 1.f, T);
}

// ------------------------------------------------------------------------------------------
// FP8 (E4M3) cache: the same attention with every cached element worth kv_scale * E4M3(code).
// ------------------------------------------------------------------------------------------
namespace {
int check_kv_scale(const char *name, float kv_scale) {
    if (!(kv_scale > 0.f) || kv_scale == INFINITY)
        return lad::set_error(LAD_EINVAL, "%s: kv_scale must be positive and finite", name);
    return LAD_OK;
}
}  // namespace

extern "C" int mla_latent_decode_fp8(const lad_bf16 *q, const uint8_t *cache, long long cache_seq_stride,
                                     float kv_scale, const int *seq_lens, const float *gate_logits, void *o,
                                     float *lse_out, int B, int Hq, int d_latent, int d_rope, int Lmax, float scale,
                                     unsigned flags, void *workspace, size_t ws_bytes, void *stream) {
    using lad::set_error;
    const char *name = "mla_latent_decode_fp8";
    int rc = check_common(name, B, Hq, d_latent, d_rope, flags, scale);
    if (rc == LAD_OK) rc = check_kv_scale(name, kv_scale);
    if (rc != LAD_OK) return rc;
    if (Lmax < 0) return set_error(LAD_EINVAL, "%s: negative Lmax", name);
    if (B == 0) return LAD_OK;
    rc = check_pointers(name, q, cache, seq_lens, o, flags);
    if (rc != LAD_OK) return rc;
    if (cache_seq_stride < static_cast<long long>(Lmax) * kDrow || cache_seq_stride % 16 != 0)
        return set_error(LAD_EINVAL, "%s: cache_seq_stride must be >= Lmax*576 and a multiple of 16", name);
    int G = 0;
    rc = sm_count_checked(name, &G);
    if (rc != LAD_OK) return rc;
    const WsLayout wl = ws_layout(B, G);
    if (!workspace || ws_bytes < wl.total || !lad::aligned(workspace, 256))
        return set_error(LAD_EWORKSPACE, "%s: workspace of %zu bytes (256-aligned) required", name, wl.total);
    CUtensorMap unused;
    std::memset(&unused, 0, sizeof unused);
    const Fp8Cache f8{cache, cache_seq_stride, Lmax};
    return run_mla(name, unused, false, PagedCache{}, nullptr, q, seq_lens, gate_logits, o, lse_out, B, scale, flags,
                   static_cast<uint8_t *>(workspace), wl, G, stream, &f8, kv_scale);
}

extern "C" int mla_latent_decode_paged_fp8(const lad_bf16 *q, const int *positions, float rope_theta,
                                           const uint8_t *kv_pages, float kv_scale, int num_pages, int page_size,
                                           const int *block_table, int block_table_stride, const int *seq_lens,
                                           const float *gate_logits, void *o, float *lse_out, int B, int Hq,
                                           int d_latent, int d_rope, float scale, unsigned flags, void *workspace,
                                           size_t ws_bytes, void *stream) {
    const char *name = "mla_latent_decode_paged_fp8";
    int rc = check_kv_scale(name, kv_scale);
    if (rc != LAD_OK) return rc;
    if (!positions)
        return run_paged(name, q, kv_pages, num_pages, page_size, block_table, block_table_stride, seq_lens,
                         gate_logits, o, lse_out, B, Hq, d_latent, d_rope, scale, flags, 0u, nullptr, workspace,
                         ws_bytes, stream, true, kv_scale);
    if (!(rope_theta > 1.f) || rope_theta == INFINITY)
        return lad::set_error(LAD_EINVAL, "%s: rope_theta must be > 1", name);
    RopeQ rq{};
    rq.positions = positions;
    rq.interleaved = (flags & LAD_FLAG_ROPE_INTERLEAVED) ? 1 : 0;
    if (d_rope == kDr) lad::rope_inverse_frequencies(static_cast<double>(rope_theta), kDr, rq.inv_freq);
    return run_paged(name, q, kv_pages, num_pages, page_size, block_table, block_table_stride, seq_lens, gate_logits,
                     o, lse_out, B, Hq, d_latent, d_rope, scale, flags, LAD_FLAG_ROPE_INTERLEAVED, &rq, workspace,
                     ws_bytes, stream, true, kv_scale);
}

// ------------------------------------------------------------------------------------------
// mla_latent_decode_noalloc: the same computation with the scratch space in a file-scope device
// array instead of a caller-provided workspace, for callers that cannot allocate device memory
// at all (for example a plugin inside a runtime that owns every device allocation, or a decode
// loop where cudaMalloc's implicit device synchronisation is not allowed).
// ------------------------------------------------------------------------------------------
namespace {

constexpr int kNoAllocMaxB = 32;    // sequences per call
constexpr int kNoAllocMaxSms = 160; // CTAs of the split kernel (one per SM)
// Partials for (SMs + B) slots plus the tile prefix: 192 x 64 x 514 x 4 B + (33 x 8 B) ~ 25.3 MB,
// held by every device that loads the library until the process exits.
constexpr size_t kNoAllocScratchBytes =
    (static_cast<size_t>(kNoAllocMaxSms + kNoAllocMaxB) * kHq * (kDl + 2) * sizeof(float) + 4 * 256 +
     (kNoAllocMaxB + 1) * sizeof(long long) + 255) / 256 * 256;

static __device__ __align__(256) uint8_t g_mla_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array, looked up once per device with that device current. The
// host-side symbol is only a stand-in and must never be handed to a kernel.
int noalloc_scratch_ptr(uint8_t **out) {
    static std::mutex mu;
    static uint8_t *ptrs[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return lad::set_error(LAD_ECUDA, "mla_latent_decode_noalloc: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return lad::set_error(LAD_EUNSUPPORTED, "mla_latent_decode_noalloc: device %d", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_mla_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return lad::set_error(LAD_ECUDA, "mla_latent_decode_noalloc: cudaGetSymbolAddress: %s",
                                  cudaGetErrorString(e));
        ptrs[dev] = static_cast<uint8_t *>(p);
    }
    *out = ptrs[dev];
    return LAD_OK;
}

}  // namespace

extern "C" size_t mla_latent_decode_noalloc_max_batch(void) { return kNoAllocMaxB; }

extern "C" int mla_latent_decode_noalloc(const lad_bf16 *q, const lad_bf16 *cache, long long cache_seq_stride,
                                         const int *seq_lens, const float *gate_logits, void *o, float *lse_out, int B,
                                         int Hq, int d_latent, int d_rope, int Lmax, float scale, unsigned flags,
                                         void *stream) {
    using lad::set_error;
    const char *name = "mla_latent_decode_noalloc";
    int rc = check_common(name, B, Hq, d_latent, d_rope, flags, scale);
    if (rc != LAD_OK) return rc;
    if (Lmax < 0) return set_error(LAD_EINVAL, "%s: negative Lmax", name);
    if (B > kNoAllocMaxB)
        return set_error(LAD_EUNSUPPORTED,
                         "%s: B = %d exceeds the built-in scratch limit of %d sequences "
                         "(use mla_latent_decode with a workspace)",
                         name, B, kNoAllocMaxB);
    if (B == 0) return LAD_OK;
    rc = check_pointers(name, q, cache, seq_lens, o, flags);
    if (rc != LAD_OK) return rc;
    if (Lmax == 0) Lmax = 1;
    if (cache_seq_stride < static_cast<long long>(Lmax) * kDrow || cache_seq_stride % 8 != 0)
        return set_error(LAD_EINVAL, "%s: cache_seq_stride must be >= Lmax*576 and a multiple of 8", name);
    const int G = lad::device_sm_count();
    if (G <= 0) return set_error(LAD_ECUDA, "%s: cannot query the SM count", name);
    if (G > kNoAllocMaxSms)
        return set_error(LAD_EUNSUPPORTED, "%s: %d SMs exceed the built-in limit of %d", name, G, kNoAllocMaxSms);
    const WsLayout wl = ws_layout(B, G);
    if (wl.total > kNoAllocScratchBytes)
        return set_error(LAD_EUNSUPPORTED, "%s: scratch of %zu bytes exceeds %zu", name, wl.total,
                         kNoAllocScratchBytes);
    uint8_t *ws = nullptr;
    rc = noalloc_scratch_ptr(&ws);
    if (rc != LAD_OK) return rc;
    CUtensorMap map_cache;
    rc = encode_contiguous(name, &map_cache, cache, B, Lmax, cache_seq_stride);
    if (rc != LAD_OK) return rc;
    return run_mla(name, map_cache, false, PagedCache{}, nullptr, q, seq_lens, gate_logits, o, lse_out, B, scale,
                   flags, ws, wl, G, stream);
}
