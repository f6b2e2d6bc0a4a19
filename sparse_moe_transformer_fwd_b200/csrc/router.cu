// Router of the MoE layer ("DeepSeek v3 and R1 Model Architecture", section
// "Local Balanced Routing to Experts": token-to-expert affinity, plus a
// per-expert bias used only to select experts).
//
// Kernel 1 (router_scores): l[t,e] = sum_i x[t,i] W_r[e,i] in binary32, one
//   fused multiply-add per term in the order i = 0..d-1 (each output is owned
//   by one thread walking d in order; no split over d, no tensor cores), then
//   s = sigmoid(l) with exp evaluated by Cody-Waite range reduction and a
//   degree-7 Taylor polynomial (W. J. Cody, W. Waite, "Software Manual for
//   the Elementary Functions", 1980).  Every operation is a correctly rounded
//   binary32 operation, so the results are reproducible bit for bit.
//   Tiling (large batches): a CTA owns 64 (or 32) tokens x 64 experts, each
//   thread 8 (or 4) tokens x 4 experts; decode-size batches use one output
//   per thread (see router_scores_small_kernel).  x and W_r chunks are staged
//   in shared memory as binary32 (bf16 widening is exact).
// Kernel 2 (router_topk): one warp per token.  sel = s + b; k rounds of a
//   warp arg-max under (sel desc, expert asc); gates g_j = s_j / S *
//   routed_scale with S the binary32 sum of the selected s in rank order.
#include "common.cuh"
#include <algorithm>
#include "kernels.h"

namespace moe {
namespace {

// ------------------------------------------------- exp / sigmoid (binary32)
// Constants derived from their definitions: ln 2 split into a head with the
// low 12 significand bits cleared (so n * head is exact for |n| < 2^12) and
// a tail; Taylor coefficients 1/i! rounded to binary32.
constexpr double kLn2 = 0.693147180559945309417232121458176568;
constexpr double kLog2e = 1.442695040888963407359924681001892137;

struct ExpConsts {
    float log2e, ln2_hi, ln2_lo, c[8];
};

__device__ __forceinline__ ExpConsts exp_consts() {
    ExpConsts k;
    k.log2e = static_cast<float>(kLog2e);
    k.ln2_hi = __uint_as_float(__float_as_uint(static_cast<float>(kLn2)) & 0xfffff000u);
    k.ln2_lo = static_cast<float>(kLn2 - static_cast<double>(k.ln2_hi));
    double f = 1.0;
    for (int i = 0; i < 8; ++i) {
        if (i) f *= i;
        k.c[i] = static_cast<float>(1.0 / f);
    }
    return k;
}

// 8 bf16 x values (one 16-byte vector) of token t at absolute column c0:
// the input itself, or the pre-norm of the residual stream h.
__device__ __forceinline__ uint4 x_vec(uint4 raw, const PreNorm &pn, int t, int c0) {
    if (!pn.gamma) return raw;
    const float r = pn.rstd[t];
    const uint4 gr = *reinterpret_cast<const uint4 *>(pn.gamma + c0);
    const uint32_t h4[4] = {raw.x, raw.y, raw.z, raw.w}, g4[4] = {gr.x, gr.y, gr.z, gr.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        o[i] = pack_bf16x2(prenorm_elem(bf16_lo(h4[i]), r, bf16_lo(g4[i])),
                           prenorm_elem(bf16_hi(h4[i]), r, bf16_hi(g4[i])));
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ float sigmoid_cw(float l, const ExpConsts &k) {
    float y = -l;
    y = fminf(fmaxf(y, -87.0f), 87.0f);
    float n = rintf(__fmul_rn(y, k.log2e));
    float r = __fmaf_rn(-n, k.ln2_hi, y);
    r = __fmaf_rn(-n, k.ln2_lo, r);
    float p = k.c[7];
#pragma unroll
    for (int i = 6; i >= 0; --i) p = __fmaf_rn(p, r, k.c[i]);
    // 2^n with n in [-126, 126]: exact scaling of a normal result
    float e = __fmul_rn(p, __int_as_float((static_cast<int>(n) + 127) << 23));
    return __fdiv_rn(1.0f, __fadd_rn(1.0f, e));
}

// ------------------------------------------------------- router_scores ---
// Larger batches: a CTA of 128 threads owns 64 (or 32) tokens x 64 experts; thread
// (ty, tx), ty < 8, tx < 16, owns tokens {4ty..4ty+3, 32+4ty..32+4ty+3} x
// experts {4tx..4tx+3}, 32 accumulators, each still a sequential FMA chain
// over d (the paired FMA of sm_100 does two independent correctly rounded
// FMAs per instruction, on experts (4tx, 4tx+1) and (4tx+2, 4tx+3)).  Per k
// step: three 16-byte shared loads (x by broadcast, W_r two wavefronts) feed
// 32 FMAs.  x and W_r chunks of 32 columns are staged transposed ([k][row],
// binary32) through registers one chunk ahead.  The 16-byte row groups of
// shared row k are XOR-swizzled by 2 * (k / 8): a thread stores 8 values of
// one row at k = 8j + c (j = 0..3), and the swizzle spreads a warp's 32
// stores (8 rows x 4 j) over all 32 banks; the compute reads stay whole
// 16-byte groups.
constexpr int RT_B = 64, RT_KC = 32, RT_THREADS = 128;
__device__ __forceinline__ int rt_swz(int k, int row) {
    return ((((row >> 2) ^ ((k >> 3) << 1)) & 15) << 2) | (row & 3);
}

// TB tokens per CTA: 64, or 32 for batches whose 64-token tiles would leave
// SMs idle (fewer tiles than SMs); each thread then owns 4 tokens, not 8.
template <int TB>
__global__ void __launch_bounds__(RT_THREADS)
router_scores_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ w, int T, int d,
                     int E, float *__restrict__ scores, PreNorm pn) {
    static_assert(TB == 64 || TB == 32, "token tile");
    constexpr int NTOK = TB / 8;                         // tokens per thread
    __shared__ __align__(16) float xs[2][RT_KC][TB];    // [k][token]
    __shared__ __align__(16) float ws[2][RT_KC][RT_B];  // [k][expert]
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int t0 = blockIdx.y * TB, e0 = blockIdx.x * RT_B;
    pdl_wait_and_trigger();

    // acc[a][j]: token a of the thread's NTOK, experts (4tx + 2j, 4tx + 2j + 1)
    float2 acc[NTOK][2];
#pragma unroll
    for (int a = 0; a < NTOK; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) acc[a][b] = make_float2(0.0f, 0.0f);

    constexpr int VPR = RT_KC / 8;                 // 16-byte vectors per row per chunk
    constexpr int NV = (TB + RT_B) * VPR;          // x rows then W_r rows
    constexpr int PER = NV / RT_THREADS;
    static_assert(NV % RT_THREADS == 0, "whole vectors per thread");
    uint4 pre[PER];
    auto load = [&](int kc) {
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int v = tid + j * RT_THREADS;
            const int row = v / VPR, col = (v % VPR) * 8;
            const bool isx = row < TB;
            const int g = isx ? t0 + row : e0 + row - TB;
            pre[j] = make_uint4(0, 0, 0, 0);
            if (g < (isx ? T : E)) {
                pre[j] = *reinterpret_cast<const uint4 *>((isx ? x : w) + static_cast<size_t>(g) * d +
                                                          kc * RT_KC + col);
                if (isx) pre[j] = x_vec(pre[j], pn, g, kc * RT_KC + col);
            }
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int v = tid + j * RT_THREADS;
            const int row = v / VPR, col = (v % VPR) * 8;
            if constexpr (TB == RT_B) {
                // x and W_r rows have the same width: one destination pointer
                float(*dst)[RT_B] = row < RT_B ? xs[buf] : ws[buf];
                const int r = row < RT_B ? row : row - RT_B;
                const uint32_t r4[4] = {pre[j].x, pre[j].y, pre[j].z, pre[j].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    dst[col + 2 * q][rt_swz(col + 2 * q, r)] = bf16_lo(r4[q]);
                    dst[col + 2 * q + 1][rt_swz(col + 2 * q + 1, r)] = bf16_hi(r4[q]);
                }
                continue;
            }
            const uint32_t r4[4] = {pre[j].x, pre[j].y, pre[j].z, pre[j].w};
            if (row < TB) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    xs[buf][col + 2 * q][rt_swz(col + 2 * q, row)] = bf16_lo(r4[q]);
                    xs[buf][col + 2 * q + 1][rt_swz(col + 2 * q + 1, row)] = bf16_hi(r4[q]);
                }
            } else {
                const int r = row - TB;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    ws[buf][col + 2 * q][rt_swz(col + 2 * q, r)] = bf16_lo(r4[q]);
                    ws[buf][col + 2 * q + 1][rt_swz(col + 2 * q + 1, r)] = bf16_hi(r4[q]);
                }
            }
        }
    };

    const int nk = d / RT_KC;
    load(0);
    store(0);
    __syncthreads();
    for (int kc = 0; kc < nk; ++kc) {
        const int buf = kc & 1;
        if (kc + 1 < nk) load(kc + 1);
        // the swizzle changes every 8 rows of k (rt_swz): per 8-row phase one
        // base address per operand, and constant offsets for its 8 rows
#pragma unroll
        for (int ph = 0; ph < RT_KC / 8; ++ph) {
            const int sw = (ph << 1) & 15;
            const float *xa_p = &xs[buf][8 * ph][((ty ^ sw) & 15) << 2];                  // tokens 4ty..
            const float *xb_p = TB == 64 ? &xs[buf][8 * ph][(((8 + ty) ^ sw) & 15) << 2]  // 32+4ty..
                                         : xa_p;
            const float *wa_p = &ws[buf][8 * ph][((tx ^ sw) & 15) << 2];                  // experts 4tx..
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float4 xa = *reinterpret_cast<const float4 *>(xa_p + u * TB);
                float4 xb = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if constexpr (TB == 64) xb = *reinterpret_cast<const float4 *>(xb_p + u * TB);
                const float4 wa = *reinterpret_cast<const float4 *>(wa_p + u * RT_B);
                const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
                const float2 wv[2] = {make_float2(wa.x, wa.y), make_float2(wa.z, wa.w)};
#pragma unroll
                for (int a = 0; a < NTOK; ++a) {
                    const float2 x2 = make_float2(xv[a], xv[a]);
#pragma unroll
                    for (int b = 0; b < 2; ++b) acc[a][b] = __ffma2_rn(x2, wv[b], acc[a][b]);
                }
            }
        }
        if (kc + 1 < nk) store(buf ^ 1);
        __syncthreads();
    }

    const ExpConsts k = exp_consts();
#pragma unroll
    for (int a = 0; a < NTOK; ++a) {
        const int t = t0 + (a < 4 ? 4 * ty + a : 32 + 4 * ty + a - 4);
        if (t >= T) continue;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int e = e0 + 4 * tx + b;
            const float l = (b & 1) ? acc[a][b >> 1].y : acc[a][b >> 1].x;
            if (e < E) scores[static_cast<size_t>(t) * E + e] = sigmoid_cw(l, k);
        }
    }
}

// ------------------------------------------------- router_scores (small T)
// Decode-sized batches: warp w of the CTA owns token t0 + w, lane l owns
// expert e0 + l; one output per thread, so the kernel is bound by the length
// of its d-long FMA chain.  Four more warps only issue the ring's cp.async
// copies: a warp issues one 16-byte-per-lane copy every ~90-160 cycles, and
// issued by the compute warps the copies took 820 of 2250 cycles per chunk
// (T = 64: 41 us -> 29 us with the copies moved off the FMA chains).  Chunks of 256 columns of the CTA's 32 W_r rows
// and BT x rows stream into a 4-stage shared-memory ring with cp.async (W_r
// rows padded by 16 bytes, so the 32 lanes' 16-byte reads of one column
// fall in distinct banks), three chunks ahead of the FMAs; each warp widens
// its own token's chunk to binary32 (applying the pre-norm if any) and the
// lanes widen W_r in registers.
constexpr int RS_KC = 256;                 // columns per chunk
constexpr int RS_WLD = RS_KC + 8;          // padded W_r row, bf16 elements
constexpr int RS_STAGES = 4;
constexpr int RS_PRODUCER_WARPS = 4;       // warps that only issue the ring's copies

template <int BT>
constexpr size_t router_small_smem() {
    return static_cast<size_t>(RS_STAGES) * (32 * RS_WLD + BT * RS_KC) * 2 +
           static_cast<size_t>(BT) * RS_KC * 4;
}

template <int BT, int NP>
__global__ void __launch_bounds__((BT + NP) * 32)
router_scores_small_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ w, int T,
                           int d, int E, float *__restrict__ scores, PreNorm pn) {
    // warps 0..BT-1 compute (one token each); warps BT..BT+NP-1 only issue the
    // cp.async copies of the ring, so the compute warps' FMA chains do not
    // wait behind the copy issue
    constexpr int NT = NP * 32;  // copy-issuing threads
    constexpr int VPR = RS_KC / 8;                    // 16-byte vectors per row per chunk
    constexpr int W_ELEMS = 32 * RS_WLD, X_ELEMS = BT * RS_KC;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint16_t *ring = reinterpret_cast<uint16_t *>(smem_raw);            // [stage][W | x]
    float *xf = reinterpret_cast<float *>(ring + RS_STAGES * (W_ELEMS + X_ELEMS));  // [BT][KC]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.y * BT, e0 = blockIdx.x * 32;
    const int t = t0 + warp, e = e0 + lane;
    const bool producer = warp >= BT;
    const int ptid = tid - BT * 32;  // index among the copy-issuing threads
    pdl_wait_and_trigger();

    const int nk = d / RS_KC;
    auto issue = [&](int kc) {
        uint16_t *ws = ring + (kc % RS_STAGES) * (W_ELEMS + X_ELEMS);
        uint16_t *xs = ws + W_ELEMS;
        for (int v = ptid; v < (32 + BT) * VPR; v += NT) {
            const int row = v / VPR, col = (v % VPR) * 8;
            if (row < 32) {
                const bool ok = e0 + row < E;
                const uint16_t *src = w + static_cast<size_t>(ok ? e0 + row : 0) * d + kc * RS_KC + col;
                cp_async16(ws + row * RS_WLD + col, src, ok);
            } else {
                const int r = row - 32;
                const bool ok = t0 + r < T;
                const uint16_t *src = x + static_cast<size_t>(ok ? t0 + r : 0) * d + kc * RS_KC + col;
                cp_async16(xs + r * RS_KC + col, src, ok);
            }
        }
    };
    if (producer) {
#pragma unroll
        for (int s = 0; s < RS_STAGES - 1; ++s) {
            if (s < nk) issue(s);
            cp_async_commit();
        }
        for (int kc = 0; kc < nk; ++kc) {
            cp_async_wait<RS_STAGES - 2>();  // this thread's copies of chunk kc landed
            __syncthreads();  // ... everyone's; and every warp is done with chunk kc - 1
            if (kc + RS_STAGES - 1 < nk) issue(kc + RS_STAGES - 1);
            cp_async_commit();
        }
        cp_async_wait<0>();
        return;
    }
    float acc = 0.0f;
    float *xw = xf + warp * RS_KC;
    for (int kc = 0; kc < nk; ++kc) {
        __syncthreads();  // chunk kc landed; every warp is done with chunk kc - 1
        const uint16_t *ws = ring + (kc % RS_STAGES) * (W_ELEMS + X_ELEMS);
        const uint16_t *xs = ws + W_ELEMS;
        // this warp's token: 8 columns per lane and pass, widened (and pre-normed)
#pragma unroll
        for (int c = lane * 8; c < RS_KC; c += 256) {
            const uint4 raw = x_vec(*reinterpret_cast<const uint4 *>(xs + warp * RS_KC + c), pn,
                                    t < T ? t : 0, kc * RS_KC + c);
            *reinterpret_cast<float4 *>(xw + c) =
                make_float4(bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y));
            *reinterpret_cast<float4 *>(xw + c + 4) =
                make_float4(bf16_lo(raw.z), bf16_hi(raw.z), bf16_lo(raw.w), bf16_hi(raw.w));
        }
        __syncwarp();
        const uint16_t *wr = ws + lane * RS_WLD;
        // operands are read two 8-column groups ahead of the FMAs that use
        // them (a 3-slot register ring, fully unrolled), so only the FMA
        // chain itself is on the critical path
        constexpr int NG = RS_KC / 8, PD = 2;
        uint4 wv[PD + 1];
        float4 xa[PD + 1], xb[PD + 1];
#pragma unroll
        for (int g = 0; g < PD; ++g) {
            wv[g] = *reinterpret_cast<const uint4 *>(wr + 8 * g);
            xa[g] = *reinterpret_cast<const float4 *>(xw + 8 * g);
            xb[g] = *reinterpret_cast<const float4 *>(xw + 8 * g + 4);
        }
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            if (g + PD < NG) {
                const int sl = (g + PD) % (PD + 1);
                wv[sl] = *reinterpret_cast<const uint4 *>(wr + 8 * (g + PD));
                xa[sl] = *reinterpret_cast<const float4 *>(xw + 8 * (g + PD));
                xb[sl] = *reinterpret_cast<const float4 *>(xw + 8 * (g + PD) + 4);
            }
            const int c = g % (PD + 1);
            acc = __fmaf_rn(xa[c].x, bf16_lo(wv[c].x), acc);
            acc = __fmaf_rn(xa[c].y, bf16_hi(wv[c].x), acc);
            acc = __fmaf_rn(xa[c].z, bf16_lo(wv[c].y), acc);
            acc = __fmaf_rn(xa[c].w, bf16_hi(wv[c].y), acc);
            acc = __fmaf_rn(xb[c].x, bf16_lo(wv[c].z), acc);
            acc = __fmaf_rn(xb[c].y, bf16_hi(wv[c].z), acc);
            acc = __fmaf_rn(xb[c].z, bf16_lo(wv[c].w), acc);
            acc = __fmaf_rn(xb[c].w, bf16_hi(wv[c].w), acc);
        }
        __syncwarp();  // xw is rewritten next chunk
    }
    if (t < T && e < E) scores[static_cast<size_t>(t) * E + e] = sigmoid_cw(acc, exp_consts());
}

// --------------------------------------------------------- router_topk ---
constexpr int kMaxPerLane = 32;  // E <= 1024

template <int PER_LANE>
__global__ void __launch_bounds__(256)
router_topk_kernel(const float *__restrict__ scores, const float *__restrict__ bias, int T, int E,
                   int k, float routed_scale, int32_t *__restrict__ idx_out,
                   float *__restrict__ gates_out) {
    pdl_wait_and_trigger();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float *srow = scores + static_cast<size_t>(t) * E;
    float s[PER_LANE], sel[PER_LANE];
    uint32_t taken = 0;
#pragma unroll
    for (int m = 0; m < PER_LANE; ++m) {
        const int e = lane + 32 * m;
        if (e < E) {
            s[m] = srow[e];
            sel[m] = __fadd_rn(s[m], bias[e]);
        } else {
            s[m] = 0.0f;
            sel[m] = 0.0f;
            taken |= 1u << m;
        }
    }
    float my_s = 0.0f;  // lane j keeps the affinity of its rank-j choice
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
        // best untaken expert of this lane (lowest index among equals: e grows with m)
        float bv = 0.0f;
        int be = 0x7fffffff;
        float bs = 0.0f;
#pragma unroll
        for (int m = 0; m < PER_LANE; ++m) {
            if (taken & (1u << m)) continue;
            const int e = lane + 32 * m;
            if (be == 0x7fffffff || sel[m] > bv) {
                bv = sel[m];
                be = e;
                bs = s[m];
            }
        }
        // warp arg-max under (sel desc, expert asc); lanes without candidates carry e = INT_MAX
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            const float os = __shfl_xor_sync(0xffffffffu, bs, off);
            const bool other_better =
                (oe != 0x7fffffff) && (be == 0x7fffffff || ov > bv || (ov == bv && oe < be));
            if (other_better) {
                bv = ov;
                be = oe;
                bs = os;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) {
            my_s = bs;
            my_e = be;
        }
    }
    // S in rank order, then the gates
    float S = 0.0f;
    for (int j = 0; j < k; ++j) S = __fadd_rn(S, __shfl_sync(0xffffffffu, my_s, j));
    if (lane < k) {
        idx_out[static_cast<size_t>(t) * k + lane] = my_e;
        gates_out[static_cast<size_t>(t) * k + lane] = __fmul_rn(__fdiv_rn(my_s, S), routed_scale);
    }
}

// Unused dynamic shared memory that caps the CTAs of a router_scores launch
// resident on one SM at `cap` (0 or 5 and more: no cap).  When the tiles of a
// launch fit in one wave, the block scheduler may stack up to five CTAs (the
// register limit) on some SMs and leave others with few; the cap spreads
// them out.  Measured at E = 256, d = 7168, 64-token tiles: T = 6144 (384
// tiles, cap 3) 0.83 -> 0.56 ms, T = 8192 (512 tiles, cap 4) 0.86 -> 0.72
// ms, T = 4096 (cap 2) unchanged; 64-token tiles so capped beat 32-token
// tiles at every T from 4096 to 16384.  Returns the padding in bytes,
// checked with the occupancy calculator (0 where the cap cannot be met), and
// remembers it per device context.
template <int TB>
int router_residency_pad(int cap) {
    if (cap <= 0 || cap >= 5) return 0;
    static DeviceConfigured configured[5]{};
    static std::atomic<int> cached[5][64];
    int dev = 0;
    cudaGetDevice(&dev);
    const bool slot = dev >= 0 && dev < 64;
    if (slot && !first_use_on_device(configured[cap])) return cached[cap][dev].load(std::memory_order_relaxed);
    int per_sm = 0, reserved = 0, opt_in = 0;
    cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    cudaDeviceGetAttribute(&opt_in, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    constexpr int kStatic = 2 * RT_KC * (TB + RT_B) * 4;  // xs and ws
    int pad = (per_sm / cap - reserved - kStatic) & ~1023;
    int n = 0;
    // the largest padding any cap uses, so a launch never exceeds the attribute
    if (pad <= 0 || kStatic + pad > opt_in) {
        pad = 0;
    } else if (cudaFuncSetAttribute(router_scores_kernel<TB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    opt_in - kStatic) != cudaSuccess ||
               cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, router_scores_kernel<TB>, RT_THREADS,
                                                             pad) != cudaSuccess) {
        cudaGetLastError();  // a refused attribute or query: launch without the cap
        pad = 0;
    } else if (n != cap) {
        pad = 0;
    }
    if (slot) {
        cached[cap][dev].store(pad, std::memory_order_relaxed);
        mark_used_on_device(configured[cap]);
    }
    return pad;
}

// Dynamic shared memory of a router_scores_small_kernel launch: the ring it
// needs, or (cap 1: no more CTAs than SMs) enough to keep a second CTA off
// each SM, so the block scheduler cannot stack two CTAs on one SM while
// others idle.  Sets the kernel's shared-memory attribute once per device
// context; -1 if even the ring cannot be granted.
int router_small_smem_for(int cap) {
    constexpr int BT = 4, NP = RS_PRODUCER_WARPS;
    constexpr int need = static_cast<int>(router_small_smem<BT>());
    static DeviceConfigured configured{};
    static std::atomic<int> cached[64];
    int dev = 0;
    cudaGetDevice(&dev);
    const bool slot = dev >= 0 && dev < 64;
    int one = 0;  // dynamic shared memory that leaves room for one CTA per SM (0: none found)
    if (slot && !first_use_on_device(configured)) {
        one = cached[dev].load(std::memory_order_relaxed);
    } else {
        int per_sm = 0, reserved = 0, opt_in = 0, n = 0;
        cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
        cudaDeviceGetAttribute(&opt_in, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (opt_in < need ||
            cudaFuncSetAttribute(router_scores_small_kernel<BT, NP>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, opt_in) != cudaSuccess) {
            cudaGetLastError();
            return -1;
        }
        const int big = std::min(opt_in, per_sm - reserved) & ~1023;
        if (big >= need) {
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, router_scores_small_kernel<BT, NP>,
                                                              (BT + NP) * 32, big) != cudaSuccess)
                cudaGetLastError();  // no cap: the query is not the caller's error
            else if (n == 1)
                one = big;
        }
        if (slot) {
            cached[dev].store(one, std::memory_order_relaxed);
            mark_used_on_device(configured);
        }
    }
    return (cap <= 1 && one > 0) ? one : need;
}

}  // namespace

cudaError_t launch_router(const uint16_t *x, const uint16_t *w, const float *bias, int T, int d,
                          int E, int k, float routed_scale, float *scores, int32_t *idx,
                          float *gates, cudaStream_t st, int *launches, PreNorm pn) {
    mark_launch(st, *launches, "router_scores");
    if (T >= 512) {
        // 64-token tiles, or 32-token tiles where 64-token tiles would leave
        // SMs without one; the CTAs resident per SM are capped at the fewest
        // that hold the whole launch in one wave (router_residency_pad)
        const int e_tiles = (E + RT_B - 1) / RT_B;
        const long long tiles64 = static_cast<long long>((T + RT_B - 1) / RT_B) * e_tiles;
        const int sms = num_sms();
        const bool wide = tiles64 >= sms;
        const long long tiles = wide ? tiles64 : static_cast<long long>((T + 31) / 32) * e_tiles;
        const int cap = static_cast<int>(std::min<long long>((tiles + sms - 1) / sms, 5));
        if (wide) {
            const int pad = router_residency_pad<64>(cap);
            dim3 grid(e_tiles, (T + 63) / 64);
            LAUNCH_OR_RETURN(launch_pdl(router_scores_kernel<64>, grid, dim3(RT_THREADS), pad, st, x, w, T,
                                        d, E, scores, pn));
        } else {
            const int pad = router_residency_pad<32>(cap);
            dim3 grid(e_tiles, (T + 31) / 32);
            LAUNCH_OR_RETURN(launch_pdl(router_scores_kernel<32>, grid, dim3(RT_THREADS), pad, st, x, w, T,
                                        d, E, scores, pn));
        }
    } else {
        constexpr int BT = 4, NP = RS_PRODUCER_WARPS;
        dim3 grid((E + 31) / 32, (T + BT - 1) / BT);
        const int ctas = static_cast<int>(grid.x * grid.y);
        const int smem = router_small_smem_for((ctas + num_sms() - 1) / num_sms());
        if (smem < 0) return cudaErrorInvalidConfiguration;
        LAUNCH_OR_RETURN(launch_pdl(router_scores_small_kernel<BT, NP>, grid, dim3((BT + NP) * 32), smem,
                                    st, x, w, T, d, E, scores, pn));
    }
    ++*launches;
    const int per_lane = (E + 31) / 32;
    dim3 grid2((T + 7) / 8);
    mark_launch(st, *launches, "router_topk");
    if (per_lane <= 1)
        LAUNCH_OR_RETURN(launch_pdl(router_topk_kernel<1>, grid2, dim3(256), 0, st, scores, bias, T, E, k, routed_scale, idx, gates));
    else if (per_lane <= 4)
        LAUNCH_OR_RETURN(launch_pdl(router_topk_kernel<4>, grid2, dim3(256), 0, st, scores, bias, T, E, k, routed_scale, idx, gates));
    else if (per_lane <= 8)
        LAUNCH_OR_RETURN(launch_pdl(router_topk_kernel<8>, grid2, dim3(256), 0, st, scores, bias, T, E, k, routed_scale, idx, gates));
    else
        LAUNCH_OR_RETURN(launch_pdl(router_topk_kernel<kMaxPerLane>, grid2, dim3(256), 0, st, scores, bias, T,
                                    E, k, routed_scale, idx, gates));
    ++*launches;
    return cudaGetLastError();
}

}  // namespace moe
