// ep.cu -- the per-rank regrouping of expert parallelism.
//
// With the N FFN experts split over G ranks (rank r holds experts [r N/G, (r+1) N/G)), each rank
// groups its own tokens' FFN picks by expert (lc_moe_permute) and sends the rows of rank r's
// experts, one contiguous slice of its grouped rows, to rank r; picks of the zero-computation
// experts never leave the rank (LongCat-Flash llm-wiki entity page, section 2.1: E_i(x) = x needs
// no expert). A receiving rank gets its rows source-major: from source 0 the rows of its local
// experts 0, 1, ... in that source's token order, then from source 1, and so on. Its grouped
// GEMMs need them expert-major. The two kernels here build that permutation and apply it:
//
//   regroup_plan_kernel  cnt[G, n_local] (rows source s sends for local expert e) ->
//                        perm[i] = arrival index of the i-th row in expert-major order
//                        (expert, then source rank, then arrival order) and the expert offsets;
//   copy_rows_kernel     dst[i] = src[map[i]] (gather) or dst[map[i]] = src[i] (scatter), rows
//                        of row_bytes bytes moved as 16-byte vectors, one warp per row.
//
// The gather puts the received rows in expert order for the GEMMs; the scatter with the same
// permutation puts the expert outputs back in arrival order, so that the return exchange (the
// inverse all-to-all) lands every output row where its source grouped the input row.
#include "common.cuh"

namespace lcmoe {

namespace {

constexpr int PLAN_THREADS = 256;
constexpr int COPY_THREADS = 256;

// Every block recomputes the small prefix tables (G * n_local <= 2048 entries) in shared memory,
// then writes the permutation entries of the (source, expert) blocks b = blockIdx.x, + gridDim.x,
// ... Block 0 also writes the expert offsets.
__global__ void __launch_bounds__(PLAN_THREADS)
    regroup_plan_kernel(const int32_t* __restrict__ cnt, int G, int n_local, int32_t* __restrict__ perm,
                        int64_t m_cap, int32_t* __restrict__ offsets, uint32_t* status) {
    extern __shared__ int32_t sm[];
    const int P = G * n_local;
    int32_t* c = sm;                  // [G][n_local] counts
    int32_t* src_in = c + P;          // [G][n_local] arrival start of block (s, e)
    int32_t* dst_in = src_in + P;     // [G][n_local] expert-major start of block (s, e)
    int32_t* src_base = dst_in + P;   // [G] arrival start of source s
    int32_t* exp_base = src_base + G; // [n_local + 1] expert-major start of expert e
    for (int i = threadIdx.x; i < P; i += blockDim.x) {
        const int v = cnt[i];
        if (v < 0) set_status(status, LC_MOE_DEV_IDX_RANGE);
        c[i] = v < 0 ? 0 : v;
    }
    __syncthreads();
    // prefix along experts within each source, and along sources within each expert
    for (int s = threadIdx.x; s < G; s += blockDim.x) {
        int run = 0;
        for (int e = 0; e < n_local; ++e) {
            src_in[s * n_local + e] = run;
            run += c[s * n_local + e];
        }
        src_base[s] = run;  // total of source s, turned into a prefix below
    }
    for (int e = threadIdx.x; e < n_local; e += blockDim.x) {
        int run = 0;
        for (int s = 0; s < G; ++s) {
            dst_in[s * n_local + e] = run;
            run += c[s * n_local + e];
        }
        exp_base[e] = run;  // total of expert e, turned into a prefix below
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int s = 0; s < G; ++s) {
            const int v = src_base[s];
            src_base[s] = run;
            run += v;
        }
        run = 0;
        for (int e = 0; e < n_local; ++e) {
            const int v = exp_base[e];
            exp_base[e] = run;
            run += v;
        }
        exp_base[n_local] = run;
        if (run > m_cap) set_status(status, LC_MOE_DEV_IDX_RANGE);
    }
    __syncthreads();
    if (blockIdx.x == 0)
        for (int e = threadIdx.x; e <= n_local; e += blockDim.x) offsets[e] = exp_base[e];
    for (int b = blockIdx.x; b < P; b += gridDim.x) {
        const int s = b / n_local, e = b - s * n_local;
        const int n = c[b];
        const int64_t from = static_cast<int64_t>(src_base[s]) + src_in[b];
        const int64_t to = static_cast<int64_t>(exp_base[e]) + dst_in[b];
        for (int j = threadIdx.x; j < n; j += blockDim.x)
            if (to + j < m_cap) perm[to + j] = static_cast<int32_t>(from + j);
    }
}

__global__ void __launch_bounds__(COPY_THREADS)
    copy_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, const int32_t* __restrict__ map,
                     int64_t n, int v16, int scatter, uint32_t* status) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (COPY_THREADS / 32);
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * (COPY_THREADS / 32) + warp; i < n; i += warps_total) {
        const int64_t m = __ldg(map + i);
        if (m < 0 || m >= n) {
            if (lane == 0) set_status(status, LC_MOE_DEV_IDX_RANGE);
            continue;
        }
        const uint4* s = src + (scatter ? i : m) * v16;
        uint4* d = dst + (scatter ? m : i) * v16;
        for (int c0 = 0; c0 < v16; c0 += 128) {  // four 16-byte loads in flight per lane
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c0 + 32 * u + lane;
                if (c < v16) v[u] = __ldg(s + c);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c0 + 32 * u + lane;
                if (c < v16) d[c] = v[u];
            }
        }
    }
}

}  // namespace

size_t regroup_plan_smem_bytes(int G, int n_local) {
    return (3 * static_cast<size_t>(G) * n_local + G + n_local + 1) * sizeof(int32_t);
}

cudaError_t launch_regroup_plan(const int32_t* cnt, int G, int n_local, int32_t* perm, int64_t m_cap,
                                int32_t* offsets, uint32_t* status, cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    // G * n_local <= 2048 keeps the tables within 33 KB, under the default 48 KB
    const size_t smem = regroup_plan_smem_bytes(G, n_local);
    int grid = G * n_local;
    if (grid > di->sm_count) grid = di->sm_count;
    regroup_plan_kernel<<<grid, PLAN_THREADS, smem, st>>>(cnt, G, n_local, perm, m_cap, offsets, status);
    return cudaGetLastError();
}

cudaError_t launch_copy_rows(const void* src, void* dst, const int32_t* map, int64_t n, int row_bytes,
                             int scatter, uint32_t* status, cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    if (n == 0) return cudaSuccess;
    int64_t blocks = (n + COPY_THREADS / 32 - 1) / (COPY_THREADS / 32);
    if (blocks > static_cast<int64_t>(di->sm_count) * 8) blocks = static_cast<int64_t>(di->sm_count) * 8;
    copy_rows_kernel<<<static_cast<int>(blocks), COPY_THREADS, 0, st>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), map, n, row_bytes / 16, scatter, status);
    return cudaGetLastError();
}

}  // namespace lcmoe
