// Permutation of the routed (token, slot) pairs into per-expert segments
// ("Local Balanced Routing to Experts": each token is assigned to experts;
// the expert GEMMs then run over contiguous per-expert segments).
//
// Deterministic counting sort in three kernels, no atomics on positions:
//  1. perm_hist: per block of 256 tokens, a shared-memory bit matrix
//     mask[e][t_local] (E x 256 bits) of which token chose which expert; per
//     expert the block count is a popcount.  The matrix is kept in the
//     workspace for kernel 3.  A repeated expert within a token or an index
//     outside [0, E) is recorded in the status word and skipped.
//  2. perm_scan: one CTA; per expert the exclusive prefix over blocks, the
//     counts, the exclusive prefix over experts (offsets), and the grouped
//     GEMM's segment/tile table (routed segments, then the shared segment).
//  3. perm_scatter: rank of token t inside expert e's segment = popcount of
//     mask[e] below t; row = offsets[e] + block prefix + rank.
// A batch of at most 256 tokens takes all three steps in one CTA
// (perm_small).  Also build_tile_table: the segment/tile table from
// caller-given offsets.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kBT = 256;          // tokens per block
constexpr int kWords = kBT / 32;  // mask words per expert per block

__global__ void __launch_bounds__(256)
perm_hist_kernel(const int32_t *__restrict__ idx, int T, int k, int E, uint32_t *__restrict__ masks,
                 int32_t *__restrict__ hist, int *status) {
    extern __shared__ uint32_t mask[];  // [E][kWords]
    const int blk = blockIdx.x;
    pdl_wait_and_trigger();
    for (int i = threadIdx.x; i < E * kWords; i += blockDim.x) mask[i] = 0;
    __syncthreads();
    const int t0 = blk * kBT;
    const int nt = min(kBT, T - t0);
    for (int i = threadIdx.x; i < nt * k; i += blockDim.x) {
        const int tl = i / k;
        const int e = idx[static_cast<size_t>(t0) * k + i];
        if (e < 0 || e >= E) {
            set_status(status, MOE_ERR_DEVICE_INDEX);
            continue;
        }
        const uint32_t bit = 1u << (tl & 31);
        const uint32_t old = atomicOr(&mask[e * kWords + (tl >> 5)], bit);
        if (old & bit) set_status(status, MOE_ERR_DEVICE_INDEX);
    }
    __syncthreads();
    uint32_t *gm = masks + static_cast<size_t>(blk) * E * kWords;
    for (int i = threadIdx.x; i < E * kWords; i += blockDim.x) gm[i] = mask[i];
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < kWords; ++w) c += __popc(mask[e * kWords + w]);
        hist[static_cast<size_t>(blk) * E + e] = c;
    }
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 1024).
__device__ int block_exclusive_scan(int v, int *tmp /* [32] */, int *total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) tmp[w] = x;
    __syncthreads();
    if (w == 0) {
        int s = tmp[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, off);
            if (lane >= off) s += y;
        }
        tmp[lane] = s;  // inclusive prefix of warp sums
    }
    __syncthreads();
    const int warp_prefix = w ? tmp[w - 1] : 0;
    const int result = warp_prefix + x - v;
    if (total) *total = tmp[31];
    __syncthreads();
    return result;
}

// Writes the segment table: seg_start[s], seg_rows[s] for s in [0, S) with
// S = E + n_shared, and tile_start[s] (S + 1 entries: prefix of m-tiles).
__device__ void write_tile_table(int count, int start, int e, int E, int T, int R, int n_shared,
                                 int tile_m, int *tmp, int32_t *seg_start, int32_t *seg_rows,
                                 int32_t *tile_start) {
    // routed segments: thread e < E; shared segment: thread E
    int rows = 0, st = 0;
    if (e < E) {
        rows = count;
        st = start;
    } else if (e == E && n_shared) {
        rows = T;
        st = R;
    }
    const int tiles = (rows + tile_m - 1) / tile_m;
    int total;
    const int ts = block_exclusive_scan(tiles, tmp, &total);
    const int S = E + n_shared;
    if (e < S) {
        seg_start[e] = st;
        seg_rows[e] = rows;
        tile_start[e] = ts;
    }
    if (e == 0) tile_start[S] = total;
}

__global__ void __launch_bounds__(1024)
perm_scan_kernel(const int32_t *__restrict__ hist, int nblk, int E, int T, int k, int n_shared,
                 int tile_m,
                 int32_t *__restrict__ blkoff, int32_t *__restrict__ counts,
                 int32_t *__restrict__ offsets, int32_t *seg_start, int32_t *seg_rows,
                 int32_t *tile_start) {
    __shared__ int tmp[32];
    const int e = threadIdx.x;
    pdl_wait_and_trigger();
    int run = 0;
    if (e < E) {
        for (int b = 0; b < nblk; ++b) {
            blkoff[static_cast<size_t>(b) * E + e] = run;
            run += hist[static_cast<size_t>(b) * E + e];
        }
        counts[e] = run;
    }
    int total;
    const int off = block_exclusive_scan(e < E ? run : 0, tmp, &total);
    if (e < E) offsets[e] = off;
    if (e == 0) offsets[E] = total;
    write_tile_table(run, off, e, E, T, T * k, n_shared, tile_m, tmp, seg_start, seg_rows, tile_start);
}

__global__ void __launch_bounds__(256)
perm_scatter_kernel(const int32_t *__restrict__ idx, int T, int k, int E,
                    const uint32_t *__restrict__ masks, const int32_t *__restrict__ blkoff,
                    const int32_t *__restrict__ offsets, int32_t *__restrict__ row_token,
                    int32_t *__restrict__ row_of) {
    extern __shared__ uint32_t mask[];  // [E][kWords]
    const int blk = blockIdx.x;
    pdl_wait_and_trigger();
    const uint32_t *gm = masks + static_cast<size_t>(blk) * E * kWords;
    for (int i = threadIdx.x; i < E * kWords; i += blockDim.x) mask[i] = gm[i];
    __syncthreads();
    const int t0 = blk * kBT;
    const int nt = min(kBT, T - t0);
    for (int i = threadIdx.x; i < nt * k; i += blockDim.x) {
        const int tl = i / k;
        const int e = idx[static_cast<size_t>(t0) * k + i];
        if (e < 0 || e >= E) continue;  // recorded by perm_hist
        const uint32_t *m = mask + e * kWords;
        int rank = 0;
        for (int w = 0; w < (tl >> 5); ++w) rank += __popc(m[w]);
        rank += __popc(m[tl >> 5] & ((1u << (tl & 31)) - 1u));
        const int row = offsets[e] + blkoff[static_cast<size_t>(blk) * E + e] + rank;
        row_token[row] = t0 + tl;
        row_of[static_cast<size_t>(t0) * k + i] = row;
    }
}

// Batches of at most 256 tokens (one bit-matrix block): kernels 1-3 in one
// CTA of 1024 threads, the bit matrix and the offsets in shared memory.
__global__ void __launch_bounds__(1024)
perm_small_kernel(const int32_t *__restrict__ idx, int T, int k, int E, int n_shared, int tile_m,
                  int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                  int32_t *__restrict__ row_token, int32_t *__restrict__ row_of,
                  int32_t *seg_start, int32_t *seg_rows, int32_t *tile_start,
                  int *status) {
    __shared__ uint32_t mask[1024 * kWords];  // [E][kWords], E <= 1024
    __shared__ int32_t off_sh[1024];
    __shared__ int tmp[32];
    const int e = threadIdx.x;
    pdl_wait_and_trigger();
    for (int i = threadIdx.x; i < E * kWords; i += blockDim.x) mask[i] = 0;
    __syncthreads();
    const int np = T * k;
    for (int i = threadIdx.x; i < np; i += blockDim.x) {
        const int v = idx[i];
        if (v < 0 || v >= E) {
            set_status(status, MOE_ERR_DEVICE_INDEX);
            continue;
        }
        const int tl = i / k;
        const uint32_t bit = 1u << (tl & 31);
        const uint32_t old = atomicOr(&mask[v * kWords + (tl >> 5)], bit);
        if (old & bit) set_status(status, MOE_ERR_DEVICE_INDEX);
    }
    __syncthreads();
    int run = 0;
    if (e < E) {
#pragma unroll
        for (int w = 0; w < kWords; ++w) run += __popc(mask[e * kWords + w]);
        counts[e] = run;
    }
    int total;
    const int off = block_exclusive_scan(e < E ? run : 0, tmp, &total);
    if (e < E) {
        offsets[e] = off;
        off_sh[e] = off;
    }
    if (e == 0) offsets[E] = total;
    write_tile_table(run, off, e, E, T, T * k, n_shared, tile_m, tmp, seg_start, seg_rows, tile_start);
    __syncthreads();
    for (int i = threadIdx.x; i < np; i += blockDim.x) {
        const int v = idx[i];
        if (v < 0 || v >= E) continue;
        const int tl = i / k;
        const uint32_t *m = mask + v * kWords;
        int rank = 0;
        for (int w = 0; w < (tl >> 5); ++w) rank += __popc(m[w]);
        rank += __popc(m[tl >> 5] & ((1u << (tl & 31)) - 1u));
        const int row = off_sh[v] + rank;
        row_token[row] = tl;
        row_of[i] = row;
    }
}

// Segment table from caller-given offsets.  A segment that is not inside
// [0, T*k) or has a negative size is recorded in the status word and
// treated as empty, so the GEMMs never touch rows outside the buffers.
__global__ void __launch_bounds__(1024)
tile_table_kernel(const int32_t *__restrict__ offsets, int E, int T, int k, int n_shared, int tile_m,
                  int32_t *seg_start, int32_t *seg_rows, int32_t *tile_start,
                  int *status) {
    __shared__ int tmp[32];
    const int e = threadIdx.x;
    pdl_wait_and_trigger();
    int count = 0, start = 0;
    if (e < E) {
        start = offsets[e];
        count = offsets[e + 1] - start;
        if (start < 0 || count < 0 || static_cast<long long>(start) + count > static_cast<long long>(T) * k) {
            set_status(status, MOE_ERR_DEVICE_INDEX);
            start = 0;
            count = 0;
        }
    }
    write_tile_table(count, start, e, E, T, T * k, n_shared, tile_m, tmp, seg_start, seg_rows, tile_start);
}

// Segment table of an expert-parallel grouped GEMM from caller segments
// (any row ranges of the receive buffer): checked copies of start, rows,
// weight slot, source rank and return row, and the prefix of tile_m-row
// tiles.  A segment that reaches outside the buffer, names a slot or a source
// that does not exist, or would return rows past its source's buffer is
// recorded in the status word and emptied.
__global__ void __launch_bounds__(1024)
ep_table_kernel(EpTableArgs a, int32_t *seg_start, int32_t *seg_rows, int32_t *tile_start,
                int32_t *seg_slot, int32_t *seg_src, int32_t *seg_ret, uint16_t **ret_y_dev,
                int *status) {
    __shared__ int tmp[32];
    const int i = threadIdx.x;
    pdl_wait_and_trigger();
    if (i < a.world) ret_y_dev[i] = a.ret_y[i];
    int start = 0, rows = 0, slot = 0, src = 0, ret = 0;
    if (i < a.n_seg) {
        start = a.start[i];
        rows = a.rows[i];
        slot = a.slot ? a.slot[i] : i;
        src = a.src[i];
        ret = a.ret[i];
        const bool ok = start >= 0 && rows >= 0 &&
                        static_cast<long long>(start) + rows <= a.rows_total && slot >= 0 &&
                        slot < a.n_slots && src >= 0 && src < a.world && ret >= 0 &&
                        static_cast<long long>(ret) + rows <= a.ret_capacity[src < 0 || src >= a.world ? 0 : src];
        if (!ok) {
            set_status(status, MOE_ERR_DEVICE_INDEX);
            start = rows = slot = src = ret = 0;
        }
    }
    const int tiles = (rows + a.tile_m - 1) / a.tile_m;
    int total;
    const int ts = block_exclusive_scan(tiles, tmp, &total);
    if (i < a.n_seg) {
        seg_start[i] = start;
        seg_rows[i] = rows;
        tile_start[i] = ts;
        seg_slot[i] = slot;
        seg_src[i] = src;
        seg_ret[i] = ret;
    }
    if (i == 0) tile_start[a.n_seg] = total;
}

}  // namespace

cudaError_t launch_permute(const int32_t *idx, int T, int k, int E, int n_shared, PermScratch s,
                           int32_t *counts, int32_t *offsets, int32_t *row_token, int32_t *row_of,
                           int *status, cudaStream_t st, int *launches) {
    const int nblk = (T + kBT - 1) / kBT;
    const size_t smem = static_cast<size_t>(E) * kWords * sizeof(uint32_t);
    if (nblk == 1) {
        mark_launch(st, *launches, "perm_small");
        LAUNCH_OR_RETURN(launch_pdl(perm_small_kernel, dim3(1), dim3(1024), 0, st, idx, T, k, E,
                                    n_shared, s.tile_m, counts, offsets, row_token, row_of, s.seg_start,
                                    s.seg_rows, s.tile_start, status));
        ++*launches;
        return cudaGetLastError();
    }
    mark_launch(st, *launches, "perm_hist");
    LAUNCH_OR_RETURN(launch_pdl(perm_hist_kernel, dim3(nblk), dim3(256), smem, st, idx, T, k, E, s.masks,
                                s.hist, status));
    ++*launches;
    mark_launch(st, *launches, "perm_scan");
    LAUNCH_OR_RETURN(launch_pdl(perm_scan_kernel, dim3(1), dim3(1024), 0, st, s.hist, nblk, E, T, k, n_shared,
                                s.tile_m, s.blkoff, counts, offsets, s.seg_start, s.seg_rows, s.tile_start));
    ++*launches;
    mark_launch(st, *launches, "perm_scatter");
    LAUNCH_OR_RETURN(launch_pdl(perm_scatter_kernel, dim3(nblk), dim3(256), smem, st, idx, T, k, E, s.masks,
                                s.blkoff, offsets, row_token, row_of));
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_tile_table(const int32_t *offsets, int E, int T, int k, int n_shared,
                              PermScratch s, int *status, cudaStream_t st, int *launches) {
    mark_launch(st, *launches, "tile_table");
    LAUNCH_OR_RETURN(launch_pdl(tile_table_kernel, dim3(1), dim3(1024), 0, st, offsets, E, T, k, n_shared,
                                s.tile_m, s.seg_start, s.seg_rows, s.tile_start, status));
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_ep_table(const EpTableArgs &a, int32_t *seg_start, int32_t *seg_rows,
                            int32_t *tile_start, int32_t *seg_slot, int32_t *seg_src,
                            int32_t *seg_ret, uint16_t **ret_y_dev, int *status, cudaStream_t st,
                            int *launches) {
    if (a.n_seg < 1 || a.n_seg > 1024 || a.world < 1 || a.world > kMaxEpRanks)
        return cudaErrorInvalidValue;
    mark_launch(st, *launches, "ep_table");
    LAUNCH_OR_RETURN(launch_pdl(ep_table_kernel, dim3(1), dim3(1024), 0, st, a, seg_start, seg_rows,
                                tile_start, seg_slot, seg_src, seg_ret, ret_y_dev, status));
    ++*launches;
    return cudaGetLastError();
}

}  // namespace moe
