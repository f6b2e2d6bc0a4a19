// Grouped expert GEMMs of the MoE layer on the 5th-generation tensor cores
// (tcgen05, sm_100a).  "DeepSeek-R1" architecture card: experts are gated
// MLPs (d_expert 2048, d_model 7168); "DeepSeek v3 and R1 Model
// Architecture", "First ever FP8 Precision...": FP8 tensor-core math;
// "DeepSeek-R1" (aguasto.com), "Quantization": blockwise FP8.
//
// One persistent kernel per GEMM, one CTA per SM, cluster size 1.
// Work item = (segment, 128-row tile of the segment, 256-column tile of B).
// Expert segments are ordered m-major, n-minor, so the CTAs running at one
// time share A tiles and the same expert's weights through L2; a single
// segment (a dense layer) is ordered n-major, m-minor, so its weight tiles are
// read from HBM once.
//   warp 0      TMA producer: A tile 128 x 128 B and two B tiles 128 x 128 B
//               (gate/up rows, or two halves of the output columns) per
//               stage, 128-byte swizzle, 4 stages.  The weights are stored in
//               128 x 128-byte tiles, so each B box is one contiguous 16 KB
//               read from HBM.
//   warp 1      TMEM allocator (512 columns) and MMA issuer (one thread):
//               tcgen05.mma M=128 N=256, K=32 (e4m3) or K=16 (bf16), four per
//               stage.
//   warps 2-3   fp32 scales: one thread fills a ring of three scale groups
//               (four K blocks of the tile's activation and weight scales)
//               in shared memory by TMA, or both warps load them where the
//               scale rows cannot be tensor-mapped; block-scaled MMA: the
//               UE8M0 scale factors for tcgen05.cp; bf16: idle
//   warps 4-11  epilogue: warp w reads TMEM lanes 32*(w%4)..+31 (tile rows);
//               warps 4-7 take columns [0,64) and [128,192), warps 8-11 take
//               [64,128) and [192,256).
// Registers: the register file is split over the SM's four sub-partitions
// and a warpgroup puts one warp on each, so warpgroup 0 drops to 40
// registers and the two epilogue warpgroups rise to 232 (setmaxnreg).
// Promotion: every 128-wide K chunk is accumulated by the tensor core into
//   one of two TMEM buffers (fresh each chunk); the epilogue loads it and adds
//   it into binary32 registers (FP8: times s_a[row, kc] * s_w[nblock, kc], the
//   per-128-K scale promotion), while the tensor core fills the other buffer.
//   BF16 takes the same path without scales, in 256-wide chunks: the tensor
//   core's internal sum over a long K is not IEEE binary32 (whole-K
//   accumulation of K = 7168 put the layer output 1.25e-3 (relative L2) away
//   from the binary64 oracle), and chunks added in binary32 registers bring
//   it back.
//   The epilogue takes each chunk's two scale products from the scale
//   ring (three 16-byte shared-memory loads per four K blocks) and issues no
//   global load in its K loop.
// Epilogue: gate/up GEMM -> H = silu(G) * U, then (FP8) 1x128 e4m3
//   quantisation of H (one 128-feature tile per row per work item; the two
//   column halves exchange their amax through shared memory; power-of-two
//   scales in the UE8M0 variant) or (BF16) bf16
//   rounding; down GEMM -> Y in bf16.  Rows past the segment end are computed
//   from neighbouring rows and never stored.  The stores transpose 16-byte
//   chunks across groups of lanes so each instruction writes whole row
//   segments.
// Every wait is bounded; on expiry the block records MOE_ERR_TIMEOUT, drains
// its own TMA loads and MMAs, frees its TMEM and exits.
#include "common.cuh"
#include "kernels.h"

#include <cstddef>
#include <cstdio>
#include <cstring>
#include <mutex>

namespace moe {
namespace {

constexpr int BM = 128;                  // tile rows
constexpr int BN = 256;                  // tile columns (TMEM columns per buffer)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * 128;        // 16 KB per stage
constexpr int B_BYTES = BN * 128;        // 32 KB per stage
constexpr int NUM_THREADS = 384;  // 3 warpgroups
constexpr int LAUNCH_REGS = 168;   // 65536 / 384, multiple of 8
constexpr int EPI_THREADS = 256;
constexpr int TMEM_COLS = 512;
constexpr int MAX_SEG = 1025;
// Block-scaled MMA: a 32-bit TMEM scale column holds four UE8M0 bytes, and an
// MMA picks one by its scale-factor id; byte j of a scale block belongs to K
// block 4g + j, so one block serves a group of four stages.
constexpr int SF_BYTES = 3 * 512;  // scale block: A, B-lo and B-hi (32 lanes x 16 bytes each)
constexpr int SF_COL = 256;        // TMEM column of the scale factors (A: 4 columns, B: 8)
constexpr int SF_GROUP = 4;        // K blocks per scale block
constexpr int SF_BUFS = 2;         // scale blocks in shared memory
constexpr int SF_STAGING = 4;      // fp32 staging slots (groups) between warps 3 and 2
constexpr int SC_GROUPS = 3;       // fp32 promotion: scale groups of four K blocks in shared memory

// Scales of the K blocks kb0 + 4g .. kb0 + 4g + 3 of one work item (K blocks
// kb0 .. kb0 + nk - 1), for the fp32 promotion: written by TMA (or by warps 2
// and 3 where the scale rows cannot be tensor-mapped), read by the epilogue.
// Row-major boxes of the [rows, K/128] and [weight rows / 128, K/128] arrays.
// Each TMA destination starts on a 128-byte boundary.
struct alignas(128) ScaleGroup {
    float a[BM][SF_GROUP];                  // activation scale: [tile row][K block % 4] (16 bytes a row)
    alignas(128) float w[2][32];            // weight scale: [column half][K block % 4] (rows 128 bytes apart)
};
constexpr int SF_AHEAD = 2;        // groups whose scale copies warp 3 keeps in flight

// Per-variant roles.  MX (block-scaled MMA): one 256-column accumulator (the
// scale factors take TMEM columns 256..267), so the epilogue drains it once
// per promotion group; warp 2 prepares the scale factors and needs a few
// more registers, taken from the epilogue.
template <bool MX>
struct Roles {
    static constexpr int NBUF = MX ? 1 : 2;              // accumulator buffers in TMEM
    static constexpr int PRODUCER_REGS = MX ? 56 : 40;   // warpgroup 0 after setmaxnreg.dec
    static constexpr int EPILOGUE_REGS = MX ? 224 : 232; // warpgroups 1-2 after setmaxnreg.inc
    static_assert(128 * PRODUCER_REGS + 256 * EPILOGUE_REGS <= NUM_THREADS * LAUNCH_REGS,
                  "register split must fit in the block's launch allocation");
};

struct __align__(1024) GemmSmem {
    uint8_t a[STAGES][A_BYTES];
    uint8_t b[STAGES][B_BYTES];
    uint8_t sf[SF_BUFS][SF_BYTES];  // MX: UE8M0 scale blocks in the tcgen05.cp source layout
    union {
        float sf_a[SF_STAGING][SF_GROUP][BM];  // MX: fp32 scales staged by warp 3 for warp 2
        ScaleGroup scg[SC_GROUPS];             // fp32 promotion: ring of scale groups
    };
    uint64_t sc_full[SC_GROUPS];   // group written (warps 2 and 3 arrive)
    uint64_t sc_empty[SC_GROUPS];  // group read (one arrive per epilogue warp)
    float sf_b[SF_STAGING][2][SF_GROUP];
    uint64_t sf_full[SF_STAGING];
    uint64_t sf_empty[SF_STAGING];
    uint64_t sf_ready[SF_BUFS];     // scale block written (warp 2 -> MMA issuer)
    uint64_t sf_free[SF_BUFS];      // scale block copied to TMEM (tcgen05.commit -> warp 2)
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t xchg[2];        // amax exchange between the two column halves
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
    float amax_x[2][2][BM];  // [iteration parity][column half][row]
    int32_t seg_start[MAX_SEG];
    int32_t seg_rows[MAX_SEG];
    int32_t tile_start[MAX_SEG + 1];
};

static_assert(sizeof(GemmSmem) + 1024 <= 227 * 1024, "shared memory budget of one CTA");
// TMA destinations of the scale ring: 128-byte boundaries
static_assert(offsetof(GemmSmem, scg) % 128 == 0 && sizeof(ScaleGroup) % 128 == 0 &&
                  offsetof(ScaleGroup, w) % 128 == 0 && sizeof(ScaleGroup::w[0]) == 128,
              "scale-group TMA destinations must start on 128-byte boundaries");

struct KParams {
    const float *a_scales;
    const float *b_scales;
    void *out;
    float *out_scales;
    const int32_t *seg_start, *seg_rows, *tile_start;
    int *status;
    int K, N_out, n_segments, b_rows, n_tiles_n;
    int inject_fault;  // 1: block 0 arms its first stage for 16 bytes that never arrive
    int ue8m0;         // H scales: power of two (UE8M0 variant) instead of amax / 448
    int rows_total;
    int mx_spc;        // MX: K blocks accumulated in TMEM per promotion into registers
    // Split K (down GEMM, software promotion only): each output tile is done
    // by ksplit work items over consecutive K-block ranges; each writes its
    // binary32 partial sums to partial[ks] (launch_splitk_reduce adds them).
    int ksplit;
    float *partial;        // [ksplit][rows_total][N_out]
    const uint16_t *residual;  // down GEMM without split: bf16 [rows_total, N_out] added before rounding Y
    int b_rowmajor;        // B row-major [slots * b_rows, K] instead of 128 x 128-byte tiles
    const int32_t *seg_slot, *seg_src, *seg_ret;
    uint16_t *const *ret_y;  // device array [world]
    int sc_tma;            // fp32 promotion: the scale groups are loaded by TMA (tmap_sa, tmap_sw)
};

template <int TM>
__device__ __forceinline__ void decode_tile(const GemmSmem &s, int n_seg, int tile, int n_tiles_n,
                                            int &seg, int &row0, int &rows_valid, int &nt) {
    if (n_seg == 1) {
        // one segment (a dense layer, or one expert): column-tile major, so the blocks that
        // run at one time take all row tiles of a few weight column tiles and
        // each weight tile is read from HBM once (row-tile major re-read the
        // dense weights once per row tile: T = 4096 layer 2.11 -> 1.71 ms);
        // the activations stay in L2
        const int m = s.tile_start[1] - s.tile_start[0];
        seg = 0;
        nt = tile / m;
        const int mloc = tile - nt * m;
        row0 = s.seg_start[0] + mloc * TM;
        rows_valid = min(TM, s.seg_rows[0] - mloc * TM);
        return;
    }
    // expert segments: row-tile major (measured better for the MoE batches)
    const int mt = tile / n_tiles_n;
    nt = tile - mt * n_tiles_n;
    int lo = 0, hi = n_seg - 1;  // last segment whose first tile is <= mt
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.tile_start[mid] <= mt) lo = mid;
        else hi = mid - 1;
    }
    seg = lo;
    const int mloc = mt - s.tile_start[seg];
    row0 = s.seg_start[seg] + mloc * TM;
    rows_valid = min(TM, s.seg_rows[seg] - mloc * TM);
}

// silu(g) = g * sigmoid(g) with the fast exponential and reciprocal: H is
// rounded to e4m3 or bf16 right after, so their few-ulp error is invisible,
// and the accurate versions made the end of every tile a long latency chain
// that stalled the tensor core (the next tile's third chunk waits for it).
// exp(-g) overflows to +inf for g < -88 and rcp(inf) = 0, so silu -> 0.
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// acc[base..base+15] (column pairs) += partial * scale (FP8 promotion) or
// += partial (BF16 chunk sum), with the paired binary32 FMA / add of sm_100
// (two correctly rounded operations per instruction).
template <bool FP8>
__device__ __forceinline__ void promote32(float2 (&acc)[64], int base, const float (&v)[32],
                                          float sc) {
    const float2 s2 = make_float2(sc, sc);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const float2 p = make_float2(v[2 * j], v[2 * j + 1]);
        if constexpr (FP8) acc[base + j] = __ffma2_rn(p, s2, acc[base + j]);
        else acc[base + j] = __fadd2_rn(acc[base + j], p);
    }
}

// Transpose of an N x N block of 16-byte chunks held by a group of N lanes
// (lanes N*g .. N*g + N-1, li = lane % N): on entry lane li holds chunks
// c[0..N-1] of its own row; on exit it holds chunk li of the group's rows
// 0..N-1 in c[0..N-1].  Each stage swaps bit m of the lane with bit m of the
// chunk index (log2 N stages of paired shuffles).  Used so that a store
// instruction writes whole row segments (N lanes x 16 bytes of one row)
// instead of 16 bytes of 32 different rows.
template <int N>
__device__ __forceinline__ void transpose_chunks(uint4 (&c)[N], int li) {
#pragma unroll
    for (int m = 1; m < N; m <<= 1) {
        const bool up = (li & m) != 0;
#pragma unroll
        for (int e = 0; e < N; ++e) {
            if (e & m) continue;
            const uint4 send = up ? c[e] : c[e | m];
            uint4 r;
            r.x = __shfl_xor_sync(0xffffffffu, send.x, m);
            r.y = __shfl_xor_sync(0xffffffffu, send.y, m);
            r.z = __shfl_xor_sync(0xffffffffu, send.z, m);
            r.w = __shfl_xor_sync(0xffffffffu, send.w, m);
            if (up) c[e] = r;
            else c[e | m] = r;
        }
    }
}

// Tile row whose output lane `l` of an epilogue warp of quadrant q stores,
// or -1 if that lane stores none (past the tile's valid rows; with 64-row
// tiles, lanes 16-31 hold the odd K steps' sums of lanes 0-15's rows).
template <bool M64>
__device__ __forceinline__ int stored_row_of_lane(int l, int q, int rows_valid) {
    const int r = M64 ? q * 16 + (l & 15) : q * 32 + l;
    return (r < rows_valid && (!M64 || l < 16)) ? r : -1;
}

// E8M0 byte of a power-of-two binary32 scale (2^-127 is the subnormal with
// exponent field 0, matching E8M0 code 0).
__device__ __forceinline__ uint32_t e8m0(float sc) { return (__float_as_uint(sc) >> 23) & 0xffu; }

template <bool FP8, bool GATE_UP, bool MX, bool M64, bool DENSE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_sa,
                    const __grid_constant__ CUtensorMap tmap_sw, const KParams p) {
    static_assert(FP8 || !MX, "the block-scaled MMA takes e4m3 operands");
    static_assert(!M64 || (FP8 && !MX), "64-row tiles: fp8 with software promotion only");
    // DENSE: the down GEMM of a dense layer, with split K (software promotion
    // only) and a residual add (a separate instance, so the expert GEMMs keep
    // their register budget)
    static_assert(!DENSE || !GATE_UP, "split K and residual: down GEMM only");
    using R = Roles<MX>;
    extern __shared__ uint8_t smem_raw[];
    GemmSmem &s = *reinterpret_cast<GemmSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = FP8 ? p.K / 128 : p.K / 64;  // stages per tile (128 bytes of K each)
    // stages per promotion chunk: FP8 128 K (the scale block); BF16 256 K;
    // MX: the tensor core applies the scales, so chunks are mx_spc K blocks
    // M64 (batches of at most 64 tokens, so every segment fits 64 rows): the
    // MMA is M = 64, which fills only lanes 16k..16k+15 of each 32-lane TMEM
    // quadrant; K steps 2p and 2p + 1 write the two lane halves of one
    // accumulator buffer, and the epilogue promotes both in one pass (each
    // thread with its own K step's scales), so the TMEM round trip is paid
    // once per two K steps.  The halves' sums are added at the tile end.
    const int SPC = MX ? p.mx_spc : (M64 ? 2 : (FP8 ? 1 : 4));
    // the epilogue multiplies each chunk by s_a * s_w (software promotion)
    constexpr bool SCALED = FP8 && !MX;
    constexpr int TM = M64 ? 64 : BM;  // rows of an MMA tile
    const int n_seg = p.n_segments;
    // work item = (output tile, K range): K blocks [kb0, kb0 + nk)
    const int KS = (DENSE && !MX) ? p.ksplit : 1;  // MX: residual only
    auto k_range = [&](int item, int &tile, int &ks, int &kb0, int &nk) {
        tile = item / KS;
        ks = item - tile * KS;
        kb0 = ks * KB / KS;
        nk = (ks + 1) * KB / KS - kb0;
    };

    // ---------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.tfull[i], 1);
            mbar_init(&s.tempty[i], EPI_THREADS / 32);
            mbar_init(&s.xchg[i], EPI_THREADS);
        }
        mbar_init(&s.mma_done, 1);
        for (int i = 0; i < SF_STAGING; ++i) {
            mbar_init(&s.sf_full[i], 1);
            mbar_init(&s.sf_empty[i], 1);
        }
        for (int i = 0; i < SC_GROUPS; ++i) {
            mbar_init(&s.sc_full[i], p.sc_tma ? 1 : 2);
            mbar_init(&s.sc_empty[i], EPI_THREADS / 32);
        }
        for (int i = 0; i < SF_BUFS; ++i) {
            mbar_init(&s.sf_ready[i], 1);
            mbar_init(&s.sf_free[i], 1);
        }
        s.abort = 0;
        fence_mbar_init();
    }
    // One segment (a dense layer): the block's first work item and the weights
    // it streams depend on no earlier kernel, so thread 0 (which initialised
    // the barriers) starts the B loads of its first `pre` stages before the
    // wait below; the producer adds their A loads after it.
    int pre = 0;
    const int NBq = p.b_rows / 128;
    auto b_blocks = [&](int slot, int nt, long long &t_lo, long long &t_hi) {
        const int nb_lo = GATE_UP ? nt : 2 * nt;
        const int nb_hi = GATE_UP ? p.N_out / 128 + nt : 2 * nt + 1;
        t_lo = static_cast<long long>(slot) * NBq + nb_lo;
        t_hi = static_cast<long long>(slot) * NBq + nb_hi;
    };
    const int rm = p.b_rowmajor;
    auto load_b = [&](void *dst, long long t, int kb, uint64_t *bar) {
        const int x = rm ? (FP8 ? kb * 128 : kb * 64) : 0;
        const int y = static_cast<int>(rm ? t * 128 : (t * KB + kb) * 128);
        tma_load_2d(dst, &tmap_b, x, y, bar);
    };
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
        const int single_items = ((p.rows_total + TM - 1) / TM) * p.n_tiles_n * KS;
        if (!p.seg_start && !MX && static_cast<int>(blockIdx.x) < single_items) {
            int tile, ks, kb0, nk;
            k_range(blockIdx.x, tile, ks, kb0, nk);
            long long t_lo, t_hi;
            b_blocks(0, tile / ((p.rows_total + TM - 1) / TM), t_lo, t_hi);  // column-tile major
            pre = min(STAGES, nk);
            for (int st = 0; st < pre; ++st) {
                mbar_arrive_expect_tx(&s.full[st], TM * 128 + B_BYTES);
                load_b(s.b[st], t_lo, kb0 + st, &s.full[st]);
                load_b(s.b[st] + B_BYTES / 2, t_hi, kb0 + st, &s.full[st]);
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(&s.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    // everything above overlaps the previous kernel; its outputs are read below
    pdl_wait_and_trigger();
    if (p.seg_start) {
        for (int i = threadIdx.x; i < n_seg; i += NUM_THREADS) {
            s.seg_start[i] = p.seg_start[i];
            s.seg_rows[i] = p.seg_rows[i];
            s.tile_start[i] = p.tile_start[i];
        }
        if (threadIdx.x == 0) s.tile_start[n_seg] = p.tile_start[n_seg];
    } else if (threadIdx.x == 0) {
        // one segment of all rows (a dense layer): no table in memory
        s.seg_start[0] = 0;
        s.seg_rows[0] = p.rows_total;
        s.tile_start[0] = 0;
        s.tile_start[1] = (p.rows_total + TM - 1) / TM;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s.tmem_base;
    const int total_tiles = s.tile_start[n_seg] * p.n_tiles_n;
    const int total_items = total_tiles * KS;
    volatile int *abort = &s.abort;

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(R::PRODUCER_REGS));
    }
    if (warp == 0) {
        // ------------------------------------------------------- producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int armed = 0;  // bit s: stage s has been armed at least once
            uint32_t armed_phase[STAGES] = {0, 0, 0, 0};
            bool ok = true;
            for (int item = blockIdx.x; item < total_items && ok; item += gridDim.x) {
                int tile, ks, kb0, nk;
                k_range(item, tile, ks, kb0, nk);
                int seg, row0, rows_valid, nt;
                decode_tile<TM>(s, n_seg, tile, p.n_tiles_n, seg, row0, rows_valid, nt);
                long long t_lo, t_hi;
                b_blocks(p.seg_slot ? __ldg(p.seg_slot + seg) : seg, nt, t_lo, t_hi);
                const bool first = item == static_cast<int>(blockIdx.x);
                for (int kb = kb0; kb < kb0 + nk; ++kb) {
                    if (!mbar_wait(&s.empty[stage], phase ^ 1, abort, p.status)) {
                        ok = false;
                        break;
                    }
                    const int kc = FP8 ? kb * 128 : kb * 64;
                    if (first && kb - kb0 < pre) {
                        // armed and its B loads issued before the wait
                        tma_load_2d(s.a[stage], &tmap_a, kc, row0, &s.full[stage]);
                    } else {
                        const bool inject = p.inject_fault && blockIdx.x == 0 && armed == 0;
                        mbar_arrive_expect_tx(&s.full[stage],
                                              TM * 128 + B_BYTES + (inject ? 16 : 0));
                        tma_load_2d(s.a[stage], &tmap_a, kc, row0, &s.full[stage]);
                        load_b(s.b[stage], t_lo, kb, &s.full[stage]);
                        load_b(s.b[stage] + B_BYTES / 2, t_hi, kb, &s.full[stage]);
                    }
                    armed |= 1 << stage;
                    armed_phase[stage] = phase;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // drain: every load this thread issued has landed before the block
            // exits (one budget for all stages)
            const long long t0 = clock64();
            for (int i = 0; i < STAGES; ++i) {
                if (!(armed & (1 << i))) continue;
                bool late = false;
                while (!mbar_try_wait(&s.full[i], armed_phase[i])) {
                    if (clock64() - t0 > kWaitBudgetCycles) {
                        set_status(p.status, MOE_ERR_TIMEOUT);
                        late = true;
                        break;
                    }
                }
                if (late) break;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            constexpr uint32_t idesc = MX ? instr_desc_mx(BM, BN) : instr_desc<FP8>(TM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int tb = 0;
            uint32_t tphase = 0;
            int gq = 0;  // MX: scale blocks consumed
            bool ok = true;
            for (int item = blockIdx.x; item < total_items && ok; item += gridDim.x) {
                int tile, ks, kb0, nk;
                k_range(item, tile, ks, kb0, nk);
                // kb counts the item's K blocks from 0 (MX: the item is all of K)
                for (int kb = 0; kb < nk; ++kb) {
                    const bool chunk_first = (kb % SPC) == 0;
                    const bool chunk_last = (kb % SPC) == SPC - 1 || kb == nk - 1;
                    if (chunk_first) {
                        if (!mbar_wait(&s.tempty[tb], tphase ^ 1, abort, p.status)) {
                            ok = false;
                            break;
                        }
                    }
                    const bool group_first = MX && (kb % SF_GROUP) == 0;
                    if (group_first &&
                        !mbar_wait(&s.sf_ready[gq % SF_BUFS], (gq / SF_BUFS) & 1, abort, p.status)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(&s.full[stage], phase, abort, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // M64: odd K steps write the upper 16 lanes of each quadrant
                    const uint32_t d_tmem = tmem_base + tb * BN +
                                            (M64 ? static_cast<uint32_t>((kb & 1) * 16) << 16 : 0u);
                    const uint64_t adesc = smem_desc_sw128(smem_u32(s.a[stage]));
                    const uint64_t bdesc = smem_desc_sw128(smem_u32(s.b[stage]));
                    if (group_first) {
                        // the group's scale block into TMEM, ordered before its MMAs
                        // and after the previous group's, which read the same columns;
                        // the commit frees the shared-memory block once it is copied
                        const int buf = gq % SF_BUFS;
                        const uint32_t sf = smem_u32(s.sf[buf]);
                        tc_cp_32x128b_warpx4(tmem_base + SF_COL, smem_desc_plain(sf, 128));
                        tc_cp_32x128b_warpx4(tmem_base + SF_COL + 4, smem_desc_plain(sf + 512, 128));
                        tc_cp_32x128b_warpx4(tmem_base + SF_COL + 8, smem_desc_plain(sf + 1024, 128));
                        tc_commit(&s.sf_free[buf]);
                        ++gq;
                    }
                    // MX: this K block's scales are byte kb % 4 of each scale column
                    // (the id in the instruction descriptor and in the TMEM address)
                    const uint32_t sid = static_cast<uint32_t>(kb % SF_GROUP);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        // +32 bytes of K per instruction: +2 in the >>4 address field;
                        // each K chunk (M64: each K step) starts a fresh partial sum
                        const uint32_t acc = ((M64 || chunk_first) && kk == 0) ? 0u : 1u;
                        if constexpr (MX)
                            tc_mma_mx(d_tmem, adesc + 2 * kk, bdesc + 2 * kk,
                                      idesc | (sid << 29) | (sid << 4),
                                      (tmem_base + SF_COL) | (sid << 30),
                                      (tmem_base + SF_COL + 4) | (sid << 30), acc);
                        else
                            tc_mma<FP8>(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, acc);
                    }
                    tc_commit(&s.empty[stage]);
                    if (chunk_last) {
                        tc_commit(&s.tfull[tb]);
                        if (++tb == R::NBUF) {
                            tb = 0;
                            tphase ^= 1;
                        }
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // all MMAs issued by this thread are complete before TMEM is freed
            tc_commit(&s.mma_done);
            long long t0 = clock64();
            while (!mbar_try_wait(&s.mma_done, 0)) {
                if (clock64() - t0 > kWaitBudgetCycles) {
                    set_status(p.status, MOE_ERR_TIMEOUT);
                    break;
                }
            }
        }
    } else if (warp == 2 || warp == 3) {
        // ------------------------------------- scale factors (block-scaled MMA)
        // Per group of four K blocks (in the producer's order): warp 3 copies
        // the fp32 scales (A's 128 rows, B's two 128-row blocks, four K blocks
        // each) from global memory into a staging ring with cp.async, SF_AHEAD
        // groups ahead; warp 2 writes their UE8M0 bytes in the tcgen05.cp
        // source layout (lane l holds rows l, 32+l, 64+l, 96+l of A, one 32-bit
        // column each, byte j for K block 4g + j) and signals the MMA issuer.
        // The split keeps global loads out of the warp that must fence its
        // shared-memory writes for the async proxy.
        if constexpr (MX) {
            const int NB = p.b_rows / 128;
            const int NG = (KB + SF_GROUP - 1) / SF_GROUP;  // groups per tile
            const int my_tiles = total_tiles > static_cast<int>(blockIdx.x)
                                     ? (total_tiles - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1
                                     : 0;
            const int n_groups = my_tiles * NG;
            bool ok = true;
            // lane 0 waits, the warp follows (bounded; false on timeout/abort)
            auto warp_wait = [&](uint64_t *bar, uint32_t parity) {
                int go = 1;
                if (lane == 0) go = mbar_wait(bar, parity, abort, p.status) ? 1 : 0;
                return __shfl_sync(0xffffffffu, go, 0) != 0;
            };
            if (warp == 3) {
                // group i: 4-byte cp.async copies into staging slot i % SF_STAGING
                // (K blocks past the end and rows past the last: zero fill), one
                // commit group per group (empty past the last one)
                auto issue = [&](int i) {
                    if (i < n_groups) {
                        const int tile = blockIdx.x + (i / NG) * gridDim.x;
                        const int kb0 = (i % NG) * SF_GROUP;
                        int seg, row0, rows_valid, nt;
                        decode_tile<TM>(s, n_seg, tile, p.n_tiles_n, seg, row0, rows_valid, nt);
                        const int slot = i % SF_STAGING;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int r = row0 + lane + 32 * c;
#pragma unroll
                            for (int j = 0; j < SF_GROUP; ++j) {
                                const bool in = r < p.rows_total && kb0 + j < KB;
                                cp_async4(&s.sf_a[slot][j][lane + 32 * c],
                                          p.a_scales + (in ? static_cast<size_t>(r) * KB + kb0 + j : 0),
                                          in);
                            }
                        }
                        if (lane < 2 * SF_GROUP) {
                            const int which = lane / SF_GROUP, j = lane % SF_GROUP;
                            const int nb = which == 0 ? (GATE_UP ? nt : 2 * nt)
                                                      : (GATE_UP ? p.N_out / 128 + nt : 2 * nt + 1);
                            const bool in = kb0 + j < KB;
                            const int slot_w = p.seg_slot ? __ldg(p.seg_slot + seg) : seg;
                            cp_async4(&s.sf_b[slot][which][j],
                                      p.b_scales + (in ? (static_cast<size_t>(slot_w) * NB + nb) * KB + kb0 + j : 0),
                                      in);
                        }
                    }
                    cp_async_commit();
                };
                auto claim = [&](int j) {  // staging slot of group j is free again
                    return j >= n_groups ||
                           warp_wait(&s.sf_empty[j % SF_STAGING], ((j / SF_STAGING) & 1) ^ 1);
                };
                for (int j = 0; j < SF_AHEAD && ok; ++j) {
                    if (!claim(j)) ok = false;
                    else issue(j);
                }
                for (int i = 0; i < n_groups && ok; ++i) {
                    if (!claim(i + SF_AHEAD)) break;
                    issue(i + SF_AHEAD);
                    cp_async_wait<SF_AHEAD>();  // group i's copies have landed
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.sf_full[i % SF_STAGING]);
                }
                cp_async_wait<0>();
            } else {
                for (int i = 0; i < n_groups; ++i) {
                    const int slot = i % SF_STAGING;
                    if (!warp_wait(&s.sf_full[slot], (i / SF_STAGING) & 1)) break;
                    uint32_t wa[4], wb[2];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t w = 0;
#pragma unroll
                        for (int j = 0; j < SF_GROUP; ++j)
                            w |= e8m0(s.sf_a[slot][j][lane + 32 * c]) << (8 * j);
                        wa[c] = w;
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t w = 0;
#pragma unroll
                        for (int j = 0; j < SF_GROUP; ++j) w |= e8m0(s.sf_b[slot][h][j]) << (8 * j);
                        wb[h] = w;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.sf_empty[slot]);
                    const int buf = i % SF_BUFS;
                    // the block's previous contents were copied to TMEM
                    if (!warp_wait(&s.sf_free[buf], ((i / SF_BUFS) & 1) ^ 1)) break;
                    uint8_t *sf = s.sf[buf];
                    *reinterpret_cast<uint4 *>(sf + 16 * lane) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
                    *reinterpret_cast<uint4 *>(sf + 512 + 16 * lane) = make_uint4(wb[0], wb[0], wb[0], wb[0]);
                    *reinterpret_cast<uint4 *>(sf + 1024 + 16 * lane) = make_uint4(wb[1], wb[1], wb[1], wb[1]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.sf_ready[buf]);
                }
            }
        } else if constexpr (SCALED) {
            // ------------------------------------ scales of the fp32 promotion
            // The epilogue's per-chunk promotion reads its scales from a ring
            // of SC_GROUPS groups in shared memory (four K blocks of the item
            // each), so the epilogue warps issue no global load.  With tensor
            // maps of the scale arrays (rows of K/128 scales a multiple of 16
            // bytes, every item's first K block a multiple of 4), one thread of
            // warp 2 fills each group with three TMA loads that complete on the
            // group's barrier: it never waits for data.
            // Otherwise warps 2 and 3 load and store the group (warp 2: rows
            // 0-63, warp 3: rows 64-127).  Either way a group is written once
            // the epilogue has released its slot.
            const int lw = warp - 2;
            const int NB = p.b_rows / 128;
            int gall = 0;  // groups written, over all items (ring position)
            bool ok = true;
            if (p.sc_tma && !(lw == 0 && lane == 0)) ok = false;  // one thread issues the loads
            for (int item = blockIdx.x; item < total_items && ok; item += gridDim.x) {
                int tile, ks, kb0, nk;
                k_range(item, tile, ks, kb0, nk);
                int seg, row0, rows_valid, nt;
                decode_tile<TM>(s, n_seg, tile, p.n_tiles_n, seg, row0, rows_valid, nt);
                const int slot_w = p.seg_slot ? __ldg(p.seg_slot + seg) : seg;
                const int nb_lo = GATE_UP ? nt : 2 * nt;
                const int nb_hi = GATE_UP ? p.N_out / 128 + nt : 2 * nt + 1;
                for (int kbg = kb0; kbg < kb0 + nk; kbg += SF_GROUP, ++gall) {
                    const int slot = gall % SC_GROUPS;
                    const uint32_t par = ((gall / SC_GROUPS) & 1) ^ 1;
                    ScaleGroup &sg = s.scg[slot];
                    if (p.sc_tma) {
                        if (!mbar_wait(&s.sc_empty[slot], par, abort, p.status)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&s.sc_full[slot], TM * 16 + 32);
                        tma_load_2d(sg.a, &tmap_sa, kbg, row0, &s.sc_full[slot]);
                        tma_load_2d(sg.w[0], &tmap_sw, kbg, slot_w * NB + nb_lo, &s.sc_full[slot]);
                        tma_load_2d(sg.w[1], &tmap_sw, kbg, slot_w * NB + nb_hi, &s.sc_full[slot]);
                        continue;
                    }
                    // lane l: rows 64 lw + l and 64 lw + 32 + l; lanes 0-7 the weight
                    // scales (lanes 0-3 the low column half, 4-7 the high)
                    const int r0 = 64 * lw + lane, r1 = r0 + 32;
                    const int wj = lane & 3, wh = (lane >> 2) & 1;
                    float a0[SF_GROUP], a1[SF_GROUP];
                    float wv = 0.0f;
#pragma unroll
                    for (int j = 0; j < SF_GROUP; ++j) {
                        const int kb = kbg + j;
                        const bool in = kb < kb0 + nk;
                        a0[j] = (in && r0 < rows_valid) ? __ldg(p.a_scales + (static_cast<size_t>(row0) + r0) * KB + kb) : 0.0f;
                        a1[j] = (in && r1 < rows_valid) ? __ldg(p.a_scales + (static_cast<size_t>(row0) + r1) * KB + kb) : 0.0f;
                    }
                    if (lane < 8 && kbg + wj < kb0 + nk)
                        wv = __ldg(p.b_scales + (static_cast<size_t>(slot_w) * NB + (wh ? nb_hi : nb_lo)) * KB + kbg + wj);
                    int go = 1;
                    if (lane == 0) go = mbar_wait(&s.sc_empty[slot], par, abort, p.status) ? 1 : 0;
                    if (__shfl_sync(0xffffffffu, go, 0) == 0) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int j = 0; j < SF_GROUP; ++j) {
                        sg.a[r0][j] = a0[j];
                        sg.a[r1][j] = a1[j];
                    }
                    if (lane < 8) sg.w[wh][wj] = wv;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.sc_full[slot]);
                }
            }
            if (p.sc_tma && lw == 0 && lane == 0) {
                // drain: the TMA loads of the last groups have landed before the
                // block exits (one budget for all)
                const long long t0 = clock64();
                for (int i = gall > SC_GROUPS ? gall - SC_GROUPS : 0; i < gall; ++i) {
                    bool late = false;
                    while (!mbar_try_wait(&s.sc_full[i % SC_GROUPS], (i / SC_GROUPS) & 1)) {
                        if (clock64() - t0 > kWaitBudgetCycles) {
                            set_status(p.status, MOE_ERR_TIMEOUT);
                            late = true;
                            break;
                        }
                    }
                    if (late) break;
                }
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------- epilogue
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(R::EPILOGUE_REGS));
        const int q = warp & 3;            // TMEM lane quadrant = tile rows 32q..32q+31
        const int half = (warp - 4) >> 2;  // column half
        // M64: lane l holds tile row 16q + l % 16 of K step parity l / 16
        const int hh = M64 ? (lane >> 4) : 0;
        const int r_in = M64 ? q * 16 + (lane & 15) : q * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        int tb = 0;
        uint32_t tphase = 0;
        int iter = 0;
        int sgrp = 0;  // scale groups of earlier items (ring position)
        bool ok = true;
        for (int item = blockIdx.x; item < total_items && ok; item += gridDim.x, ++iter) {
            int tile, ks, kb0, nk;
            k_range(item, tile, ks, kb0, nk);
            const int nch = (nk + SPC - 1) / SPC;  // K chunks of the item (last may be short)
            int seg, row0, rows_valid, nt;
            decode_tile<TM>(s, n_seg, tile, p.n_tiles_n, seg, row0, rows_valid, nt);
            const bool warp_active = q * (M64 ? 16 : 32) < rows_valid;
            const bool valid = r_in < rows_valid;
            const bool store_row = valid && hh == 0;  // M64: one lane of the pair stores
            const size_t row = static_cast<size_t>(row0) + r_in;
            const int col_lo = half * 64, col_hi = 128 + half * 64;
            float2 acc2[64];  // columns (2j, 2j+1) of the thread's 128
#pragma unroll
            for (int i = 0; i < 64; ++i) acc2[i] = make_float2(0.0f, 0.0f);
            // K block (counted from kb0) whose partial this thread promotes in chunk c
            auto kb_of = [&](int c) { return M64 ? 2 * c + hh : c; };
            // chunks per scale group of four K blocks (M64: K steps 2c and
            // 2c + 1 share a chunk, so a group is two chunks)
            constexpr int GPC = M64 ? 2 : 4;
            // Scales from the ring in shared memory, read a group (four K
            // blocks) at a time with three 16-byte shared-memory loads: at the
            // end of the chunk before the group's first (after that chunk's
            // buffer release) and consumed only after the next TMEM loads have
            // landed, so shared-memory latency stays off the accumulator round
            // trip.  The previous group's slot is released at that read (its
            // values were consumed a chunk earlier), the item's last group
            // after the item.
            float4 g_a = make_float4(0.0f, 0.0f, 0.0f, 0.0f), g_wl = g_a, g_wh = g_a;
            auto fetch_scales = [&](int cc) {
                if (cc % GPC != 0) return true;
                const int gi = sgrp + cc / GPC;
                const int slot = gi % SC_GROUPS;
                if (cc > 0) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.sc_empty[(gi - 1) % SC_GROUPS]);
                }
                if (!mbar_wait(&s.sc_full[slot], (gi / SC_GROUPS) & 1, abort, p.status)) return false;
                g_a = *reinterpret_cast<const float4 *>(s.scg[slot].a[r_in]);
                g_wl = *reinterpret_cast<const float4 *>(s.scg[slot].w[0]);
                g_wh = *reinterpret_cast<const float4 *>(s.scg[slot].w[1]);
                return true;
            };
            auto pick = [](const float4 &v, int j) { return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w)); };
            if constexpr (SCALED) ok = fetch_scales(0);
            for (int c = 0; c < nch && ok; ++c) {
                const bool kvalid = !M64 || kb_of(c) < nk;  // M64, odd K: no partial in the upper half
                if (!mbar_wait(&s.tfull[tb], tphase, abort, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // four 32-column pieces, two loads in flight at a time; the
                // buffer is released as soon as the last piece is in registers
                // (before its FMAs), since the MMA two chunks ahead waits for it
                float va[32], vb[32];
                float sc_lo = 1.0f, sc_hi = 1.0f;
                const bool add = warp_active && kvalid;  // the loads below are warp-wide
                if (warp_active) {
                    const uint32_t base = lane_base + tb * BN;
                    tmem_ld32(base + col_lo, va);
                    tmem_ld32(base + col_lo + 32, vb);
                    tmem_wait_ld(va, vb);
                    if constexpr (SCALED) {
                        // the group's scale loads are consumed here, not earlier
                        asm volatile("" : "+f"(g_a.x), "+f"(g_a.y), "+f"(g_a.z), "+f"(g_a.w));
                        const int j = kb_of(c) & 3;
                        const float sa = pick(g_a, j);
                        sc_lo = sa * pick(g_wl, j);
                        sc_hi = sa * pick(g_wh, j);
                    }
                    if (add) promote32<SCALED>(acc2, 0, va, sc_lo);
                    tmem_ld32(base + col_hi, va);
                    if (add) promote32<SCALED>(acc2, 16, vb, sc_lo);
                    tmem_ld32(base + col_hi + 32, vb);
                    tmem_wait_ld(va, vb);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.tempty[tb]);
                if (add) {
                    promote32<SCALED>(acc2, 32, va, sc_hi);
                    promote32<SCALED>(acc2, 48, vb, sc_hi);
                }
                if (SCALED && c + 1 < nch && !fetch_scales(c + 1)) ok = false;
                if (++tb == R::NBUF) {
                    tb = 0;
                    tphase ^= 1;
                }
            }
            if constexpr (SCALED) {
                // the item's last scale group has been consumed
                __syncwarp();
                const int n_groups = (nk + SF_GROUP - 1) / SF_GROUP;
                if (ok && lane == 0) mbar_arrive(&s.sc_empty[(sgrp + n_groups - 1) % SC_GROUPS]);
                sgrp += n_groups;
            }
            if (!ok) break;
            if constexpr (M64) {
                // even and odd K steps' sums of the same row meet (both lanes get
                // the same total)
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    acc2[i].x += __shfl_xor_sync(0xffffffffu, acc2[i].x, 16);
                    acc2[i].y += __shfl_xor_sync(0xffffffffu, acc2[i].y, 16);
                }
            }
            // column c of the thread's 128 (in place, no copy)
            auto acc = [&](int c) -> float & { return (c & 1) ? acc2[c >> 1].y : acc2[c >> 1].x; };
            if constexpr (GATE_UP) {
                // H = silu(G) * U for features nt*128 + half*64 + c, c < 64
                // (warps without valid rows skip the math, not the exchange)
                float m = 0.0f;
                if (warp_active) {
#pragma unroll
                    for (int c = 0; c < 64; ++c) {
                        acc(c) = silu(acc(c)) * acc(64 + c);
                        m = fmaxf(m, fabsf(acc(c)));
                    }
                }
                if constexpr (FP8) {
                    const int par = iter & 1;
                    s.amax_x[par][half][r_in] = m;
                    mbar_arrive(&s.xchg[par]);
                    if (!mbar_wait(&s.xchg[par], (iter >> 1) & 1, abort, p.status)) {
                        ok = false;
                        break;
                    }
                    const float amax = fmaxf(m, s.amax_x[par][half ^ 1][r_in]);
                    float sc = 1.0f, inv = 0.0f;
                    if (amax != 0.0f) {
                        if (p.ue8m0) {
                            sc = ue8m0_scale(amax, &inv);
                        } else {
                            sc = __fdiv_rn(amax, 448.0f);
                            inv = __fdiv_rn(448.0f, amax);
                        }
                    }
                    if (warp_active) {  // uniform over the warp
                        // 64 codes = four 16-byte chunks; transposed across
                        // groups of 4 lanes so each store writes 64 contiguous
                        // bytes of a row
                        uint4 ch[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            uint32_t w[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int b = 16 * c + 4 * i;
                                const uint32_t lo = e4m3x2(__fmul_rn(acc(b), inv), __fmul_rn(acc(b + 1), inv));
                                const uint32_t hi = e4m3x2(__fmul_rn(acc(b + 2), inv), __fmul_rn(acc(b + 3), inv));
                                w[i] = amax != 0.0f ? (lo | (hi << 16)) : 0u;
                            }
                            ch[c] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                        const int li = lane & 3;
                        transpose_chunks<4>(ch, li);
                        uint8_t *h0 = static_cast<uint8_t *>(p.out) + static_cast<size_t>(row0) * p.N_out +
                                      nt * 128 + half * 64 + 16 * li;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int o = stored_row_of_lane<M64>((lane & ~3) | j, q, rows_valid);
                            if (o >= 0) *reinterpret_cast<uint4 *>(h0 + static_cast<size_t>(o) * p.N_out) = ch[j];
                        }
                    }
                    if (store_row && half == 0) p.out_scales[row * (p.N_out / 128) + nt] = sc;
                } else if (warp_active) {
                    // bf16 H: 64 values = eight 16-byte chunks, transposed as Y
                    uint4 ch[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int c = 8 * j;
                        ch[j] = make_uint4(pack_bf16x2(acc(c), acc(c + 1)), pack_bf16x2(acc(c + 2), acc(c + 3)),
                                           pack_bf16x2(acc(c + 4), acc(c + 5)), pack_bf16x2(acc(c + 6), acc(c + 7)));
                    }
                    const int li = lane & 7;
                    transpose_chunks<8>(ch, li);
                    uint16_t *h0 = static_cast<uint16_t *>(p.out) + static_cast<size_t>(row0) * p.N_out +
                                   nt * 128 + half * 64 + 8 * li;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int o = stored_row_of_lane<M64>((lane & ~7) | j, q, rows_valid);
                        if (o >= 0) *reinterpret_cast<uint4 *>(h0 + static_cast<size_t>(o) * p.N_out) = ch[j];
                    }
                }
            } else {
                if (DENSE && KS > 1) {
                    // split K: store this K range's binary32 partial sums; the
                    // reduce kernel that follows adds the KS ranges in K order
                    ks = item - (item / KS) * KS;  // recomputed: not kept live through the chunk loop
                    if (store_row) {
                        float *pp = p.partial + (static_cast<size_t>(ks) * p.rows_total + row) * p.N_out + nt * 256;
#pragma unroll
                        for (int c = 0; c < 64; c += 4) {
                            *reinterpret_cast<float4 *>(pp + col_lo + c) =
                                make_float4(acc(c), acc(c + 1), acc(c + 2), acc(c + 3));
                            *reinterpret_cast<float4 *>(pp + col_hi + c) =
                                make_float4(acc(64 + c), acc(64 + c + 1), acc(64 + c + 2), acc(64 + c + 3));
                        }
                    }
                    continue;
                }
                if (!warp_active) continue;  // uniform over the warp
                if (DENSE && p.residual && store_row) {
                    // the pre-norm block's residual, added before the one rounding
                    const uint16_t *rp = p.residual + row * p.N_out + nt * 256;
#pragma unroll
                    for (int c = 0; c < 64; c += 8) {
                        const uint4 a = *reinterpret_cast<const uint4 *>(rp + col_lo + c);
                        const uint4 b = *reinterpret_cast<const uint4 *>(rp + col_hi + c);
                        const uint32_t ra[4] = {a.x, a.y, a.z, a.w}, rb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            acc(c + 2 * i) = __fadd_rn(acc(c + 2 * i), bf16_lo(ra[i]));
                            acc(c + 2 * i + 1) = __fadd_rn(acc(c + 2 * i + 1), bf16_hi(ra[i]));
                            acc(64 + c + 2 * i) = __fadd_rn(acc(64 + c + 2 * i), bf16_lo(rb[i]));
                            acc(64 + c + 2 * i + 1) = __fadd_rn(acc(64 + c + 2 * i + 1), bf16_hi(rb[i]));
                        }
                    }
                }
                // Y rows of the tile: one segment, so the base is uniform over
                // the warp and each lane's row differs by its index
                uint16_t *ybase = static_cast<uint16_t *>(p.out) + nt * 256;
                long long yr = static_cast<long long>(row);
                if (p.seg_ret) {
                    // expert parallelism: straight into the source rank's Y buffer
                    ybase = p.ret_y[__ldg(p.seg_src + seg)] + nt * 256;
                    yr = static_cast<long long>(__ldg(p.seg_ret + seg)) + (yr - s.seg_start[seg]);
                }
                // bf16 chunks of 8 columns; transposed across groups of 8
                // lanes so each store writes 128 contiguous bytes of a row
                // (one 64-column half at a time, to bound the live registers)
                const long long yr0 = yr - r_in;
                const int li = lane & 7;
                int yoff[8];  // tile row held by lane (lane & ~7) | j, -1: not stored
#pragma unroll
                for (int j = 0; j < 8; ++j) yoff[j] = stored_row_of_lane<M64>((lane & ~7) | j, q, rows_valid);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint4 ch[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int c = 64 * hf + 8 * j;
                        ch[j] = make_uint4(pack_bf16x2(acc(c), acc(c + 1)), pack_bf16x2(acc(c + 2), acc(c + 3)),
                                           pack_bf16x2(acc(c + 4), acc(c + 5)), pack_bf16x2(acc(c + 6), acc(c + 7)));
                    }
                    transpose_chunks<8>(ch, li);
                    const int col = (hf ? col_hi : col_lo) + 8 * li;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (yoff[j] >= 0)
                            *reinterpret_cast<uint4 *>(ybase + (yr0 + yoff[j]) * p.N_out + col) = ch[j];
                }
            }
        }
    }

    // ------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ----------------------------------------------------------- host side ---
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

bool make_map_2d(CUtensorMap *m, const void *base, bool fp8, int K, int rows, int box_rows = 128) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const int es = fp8 ? 1 : 2;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * es};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / es), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
               const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// binary32 [rows, cols] row-major, boxes of box_rows x 4 (16 bytes a row, no
// swizzle; reads past the array give 0)
bool make_map_scales(CUtensorMap *m, const float *base, int cols, long long rows, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || cols % 4 != 0 || (reinterpret_cast<uintptr_t>(base) & 15) != 0 || rows < 1 ||
        rows >= (1LL << 31))
        return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 4};
    cuuint32_t box[2] = {4, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool FP8, bool GATE_UP, bool MX, bool M64 = false, bool DENSE = false>
cudaError_t launch_t(const CUtensorMap &ma, const CUtensorMap &mb, const CUtensorMap &msa,
                     const CUtensorMap &msw, const KParams &kp, int grid, cudaStream_t st) {
    const size_t smem = sizeof(GemmSmem) + 1024;
    static DeviceConfigured configured{};  // per template instance
    if (first_use_on_device(configured)) {
        // setmaxnreg redistributes exactly NUM_THREADS * LAUNCH_REGS registers:
        // refuse to launch a build whose register count differs, as the
        // epilogue's increase would then never be granted.
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, grouped_gemm_kernel<FP8, GATE_UP, MX, M64, DENSE>);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != LAUNCH_REGS) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(grouped_gemm_kernel<FP8, GATE_UP, MX, M64, DENSE>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        mark_used_on_device(configured);
    }
    return launch_pdl(grouped_gemm_kernel<FP8, GATE_UP, MX, M64, DENSE>, dim3(grid), dim3(NUM_THREADS), smem, st,
                      ma, mb, msa, msw, kp);
}

}  // namespace

cudaError_t launch_grouped_gemm(const GemmArgs &g, cudaStream_t st, int *launches) {
    if (g.n_segments > MAX_SEG) return cudaErrorInvalidValue;
    const int b_rows = g.gate_up ? 2 * g.N_out : g.N_out;
    CUtensorMap ma, mb;
    // 64-row MMA tiles: the segment table counts 64-row tiles (fp32 scales)
    const bool m64 = g.tile_m == 64;
    if (m64 && (!g.fp8 || g.ue8m0)) return cudaErrorInvalidValue;
    if (!m64 && g.tile_m != 128) return cudaErrorInvalidValue;
    if (!make_map_2d(&ma, g.a, g.fp8, g.K, g.rows_total, m64 ? 64 : 128))
        return cudaErrorInvalidValue;
    if (g.b_rowmajor) {
        const long long rows = static_cast<long long>(g.n_slots) * b_rows;
        if (rows >= (1LL << 31)) return cudaErrorInvalidValue;
        if (!make_map_2d(&mb, g.b, g.fp8, g.K, static_cast<int>(rows))) return cudaErrorInvalidValue;
    } else {
        const long long b_tile_rows = static_cast<long long>(g.n_slots) * b_rows * (g.K * (g.fp8 ? 1 : 2) / 128);
        if (b_tile_rows >= (1LL << 31)) return cudaErrorInvalidValue;
        if (!make_map_2d(&mb, g.b, g.fp8, g.fp8 ? 128 : 64, static_cast<int>(b_tile_rows)))
            return cudaErrorInvalidValue;
    }
    KParams kp{};
    kp.a_scales = g.a_scales;
    kp.b_scales = g.b_scales;
    kp.out = g.out;
    kp.out_scales = g.out_scales;
    kp.seg_start = g.seg_start;
    kp.seg_rows = g.seg_rows;
    kp.tile_start = g.tile_start;
    kp.status = g.status;
    kp.K = g.K;
    kp.N_out = g.N_out;
    kp.n_segments = g.n_segments;
    kp.b_rows = b_rows;
    kp.n_tiles_n = g.gate_up ? g.N_out / 128 : g.N_out / 256;
    kp.inject_fault = g.inject_fault;
    kp.ue8m0 = g.ue8m0 ? 1 : 0;
    kp.rows_total = g.rows_total;
    kp.b_rowmajor = g.b_rowmajor ? 1 : 0;
    kp.seg_slot = g.seg_slot;
    kp.seg_src = g.seg_src;
    kp.seg_ret = g.seg_ret;
    kp.ret_y = g.ret_y_dev;
    if (g.seg_ret && !g.ret_y_dev) return cudaErrorInvalidValue;
    // fp32 promotion: tensor maps of the two scale arrays when their rows are
    // whole 16-byte units (else warps 2 and 3 load the scale groups)
    CUtensorMap msa, msw;
    std::memset(&msa, 0, sizeof(msa));
    std::memset(&msw, 0, sizeof(msw));
    if (g.fp8 && !g.ue8m0) {
        const int kbn = g.K / 128;
        const int ksp = (g.gate_up || g.ksplit < 1) ? 1 : g.ksplit;
        bool aligned = true;  // every work item's first K block a multiple of 4 (16-byte x)
        for (int ks = 0; ks < ksp; ++ks) aligned = aligned && (ks * kbn / ksp) % 4 == 0;
        kp.sc_tma = aligned &&
                    make_map_scales(&msa, g.a_scales, kbn, g.rows_total, m64 ? 64 : 128) &&
                    make_map_scales(&msw, g.b_scales, kbn, static_cast<long long>(g.n_slots) * (b_rows / 128), 1)
                        ? 1 : 0;
    }
    // block-scaled MMA (UE8M0 scales): all of K accumulates in TMEM
    kp.mx_spc = g.K / 128;
    const bool mx = g.fp8 && g.ue8m0;
    kp.ksplit = (g.gate_up || mx || g.ksplit < 1) ? 1 : g.ksplit;
    if (kp.ksplit > 1 && (!g.partial || kp.ksplit > (g.fp8 ? g.K / 128 : g.K / 64)))
        return cudaErrorInvalidValue;
    kp.partial = g.partial;
    // with split K the residual is added by the reduce kernel
    kp.residual = (g.gate_up || kp.ksplit > 1) ? nullptr : g.residual;
    // upper bound of work items: every segment's tiles, each at most one partial
    const long long max_mtiles = g.rows_total / g.tile_m + g.n_segments;
    const long long max_tiles = max_mtiles * kp.n_tiles_n * kp.ksplit;
    const int grid = static_cast<int>(max_tiles < num_sms() ? max_tiles : num_sms());
    if (grid <= 0) return cudaSuccess;
    cudaError_t e;
    mark_launch(st, *launches, g.gate_up ? "grouped_gemm_gate_up" : "grouped_gemm_down");
    // the dense layer's down GEMM (split K or a residual) has its own instances
    const bool dense = !g.gate_up && (kp.ksplit > 1 || kp.residual);
    if (dense && mx)
        e = launch_t<true, false, true, false, true>(ma, mb, msa, msw, kp, grid, st);
    else if (g.fp8 && g.ue8m0)
        e = g.gate_up ? launch_t<true, true, true>(ma, mb, msa, msw, kp, grid, st)
                      : launch_t<true, false, true>(ma, mb, msa, msw, kp, grid, st);
    else if (dense && g.fp8 && m64)
        e = launch_t<true, false, false, true, true>(ma, mb, msa, msw, kp, grid, st);
    else if (dense && g.fp8)
        e = launch_t<true, false, false, false, true>(ma, mb, msa, msw, kp, grid, st);
    else if (dense)
        e = launch_t<false, false, false, false, true>(ma, mb, msa, msw, kp, grid, st);
    else if (g.fp8 && m64)
        e = g.gate_up ? launch_t<true, true, false, true>(ma, mb, msa, msw, kp, grid, st)
                      : launch_t<true, false, false, true>(ma, mb, msa, msw, kp, grid, st);
    else if (g.fp8)
        e = g.gate_up ? launch_t<true, true, false>(ma, mb, msa, msw, kp, grid, st)
                      : launch_t<true, false, false>(ma, mb, msa, msw, kp, grid, st);
    else
        e = g.gate_up ? launch_t<false, true, false>(ma, mb, msa, msw, kp, grid, st)
                      : launch_t<false, false, false>(ma, mb, msa, msw, kp, grid, st);
    ++*launches;
    return e;
}

// ------------------------------------------------------- split-K reduce ---
namespace {

// out[r, n] = bf16( ((partial[0][r][n] + partial[1][r][n]) + ...) (+ residual) ),
// binary32 adds in K-range order; one thread per 8 columns, every K range's
// loads issued before the adds.
__global__ void __launch_bounds__(128)
splitk_reduce_kernel(const float *__restrict__ partial, int ksplit, int rows, int n,
                     const uint16_t *__restrict__ residual, uint16_t *__restrict__ out) {
    const int r = blockIdx.x;
    const int v = blockIdx.y * blockDim.x + threadIdx.x;  // 8-column group
    pdl_wait_and_trigger();
    if (v >= n / 8) return;
    const size_t off = static_cast<size_t>(r) * n + static_cast<size_t>(v) * 8;
    const size_t kstride = static_cast<size_t>(rows) * n;
    float4 a[8], b[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (k < ksplit) {
            a[k] = __ldcg(reinterpret_cast<const float4 *>(partial + k * kstride + off));
            b[k] = __ldcg(reinterpret_cast<const float4 *>(partial + k * kstride + off + 4));
        }
    }
    float f[8] = {a[0].x, a[0].y, a[0].z, a[0].w, b[0].x, b[0].y, b[0].z, b[0].w};
#pragma unroll
    for (int k = 1; k < 8; ++k) {
        if (k < ksplit) {
            const float g[8] = {a[k].x, a[k].y, a[k].z, a[k].w, b[k].x, b[k].y, b[k].z, b[k].w};
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = __fadd_rn(f[i], g[i]);
        }
    }
    if (residual) {
        const uint4 h = *reinterpret_cast<const uint4 *>(residual + off);
        const uint32_t w[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __fadd_rn(f[2 * i], bf16_lo(w[i]));
            f[2 * i + 1] = __fadd_rn(f[2 * i + 1], bf16_hi(w[i]));
        }
    }
    uint4 o;
    o.x = pack_bf16x2(f[0], f[1]);
    o.y = pack_bf16x2(f[2], f[3]);
    o.z = pack_bf16x2(f[4], f[5]);
    o.w = pack_bf16x2(f[6], f[7]);
    *reinterpret_cast<uint4 *>(out + off) = o;
}

}  // namespace

cudaError_t launch_splitk_reduce(const float *partial, int ksplit, int rows, int n,
                                 const uint16_t *residual, uint16_t *out, cudaStream_t st,
                                 int *launches) {
    if (ksplit < 1 || ksplit > kMaxSplitK || n % 8) return cudaErrorInvalidValue;
    mark_launch(st, *launches, "splitk_reduce");
    const dim3 grid(rows, (n / 8 + 127) / 128);
    LAUNCH_OR_RETURN(launch_pdl(splitk_reduce_kernel, grid, dim3(128), 0, st, partial, ksplit,
                                rows, n, residual, out));
    ++*launches;
    return cudaGetLastError();
}

}  // namespace moe
