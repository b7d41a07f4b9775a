// permute.cu -- grouping of the (token, pick) pairs routed to FFN experts, and the row gather.
//
// Only the N FFN experts of the MoE equation (LongCat-Flash llm-wiki entity page, section 2.1)
// do work; picks of the Z zero-computation experts (ids >= N) get no row, so they are never
// copied, multiplied or written back (the combine adds their g x_t term directly).
//
// Deterministic stable counting sort, no atomics on positions:
//   count   : block b owns tokens [256 b, 256 b + 256). For each FFN expert e it builds a 256-bit
//             mask of the block's tokens that picked e (atomicOr in shared memory: order-free),
//             and writes the block count popc(mask) to cnt[b][e].
//   scan    : one block; for each expert a running sum over blocks gives base[b][e] (rows of e in
//             earlier blocks), then an exclusive scan over experts gives offsets[e].
//   scatter : the row of pick (t, r) of expert e is
//             offsets[e] + base[b][e] + popc(mask of e restricted to tokens before t in block b),
//             so rows of an expert are in ascending token order. Writes pair_row and row_token.
//   single  : a batch of at most 256 tokens (one block) does all three in one launch.
//   gather  : per token, x_t is read once into shared memory with one bulk async copy and
//             written to each of its FFN rows with one bulk store per row (rows above 25 KB:
//             one warp per token copies 16-byte vectors through registers); x_t is read once
//             however many FFN experts the token picked.
#include <mutex>

#include "common.cuh"

namespace lcmoe {

namespace {

constexpr int PB = 256;          // tokens per block = threads per block
constexpr int MASK_WORDS = PB / 32;

__device__ __forceinline__ bool build_masks(const int32_t* __restrict__ idx, int T, int K, int N,
                                            int E, uint32_t* mask, uint32_t* status) {
    const int t = blockIdx.x * PB + threadIdx.x;
    bool bad = false;
    if (t < T) {
        const uint32_t bit = 1u << (threadIdx.x & 31);
        const int w = threadIdx.x >> 5;
        for (int r = 0; r < K; ++r) {
            const int e = idx[static_cast<int64_t>(t) * K + r];
            if (e < 0 || e >= E) {
                bad = true;
            } else if (e < N) {
                const uint32_t old = atomicOr(&mask[e * MASK_WORDS + w], bit);
                if (old & bit) set_status(status, LC_MOE_DEV_DUP_PICK);
            }
        }
    }
    return bad;
}

__global__ void __launch_bounds__(PB)
    perm_count_kernel(const int32_t* __restrict__ idx, int T, int K, int N, int E,
                      int32_t* __restrict__ cnt, uint32_t* __restrict__ status) {
    extern __shared__ uint32_t mask[];
    for (int i = threadIdx.x; i < N * MASK_WORDS; i += PB) mask[i] = 0;
    __syncthreads();
    const bool bad = build_masks(idx, T, K, N, E, mask, status);
    if (__syncthreads_or(bad) && threadIdx.x == 0) set_status(status, LC_MOE_DEV_IDX_RANGE);
    for (int e = threadIdx.x; e < N; e += PB) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < MASK_WORDS; ++w) c += __popc(mask[e * MASK_WORDS + w]);
        cnt[static_cast<int64_t>(blockIdx.x) * N + e] = c;
    }
}

constexpr int SCAN_THREADS = 1024;

__global__ void __launch_bounds__(SCAN_THREADS)
    perm_scan_kernel(const int32_t* __restrict__ cnt, int nblk, int N, int32_t* __restrict__ base,
                     int32_t* __restrict__ offsets) {
    extern __shared__ int32_t tot[];  // [N]
    __shared__ int32_t warp_sums[SCAN_THREADS / 32];
    __shared__ int32_t carry;
    for (int e = threadIdx.x; e < N; e += SCAN_THREADS) {
        int run = 0;
        int b = 0;
        for (; b + 4 <= nblk; b += 4) {
            const int c0 = cnt[static_cast<int64_t>(b) * N + e];
            const int c1 = cnt[static_cast<int64_t>(b + 1) * N + e];
            const int c2 = cnt[static_cast<int64_t>(b + 2) * N + e];
            const int c3 = cnt[static_cast<int64_t>(b + 3) * N + e];
            base[static_cast<int64_t>(b) * N + e] = run;
            base[static_cast<int64_t>(b + 1) * N + e] = run + c0;
            base[static_cast<int64_t>(b + 2) * N + e] = run + c0 + c1;
            base[static_cast<int64_t>(b + 3) * N + e] = run + c0 + c1 + c2;
            run += c0 + c1 + c2 + c3;
        }
        for (; b < nblk; ++b) {
            const int c = cnt[static_cast<int64_t>(b) * N + e];
            base[static_cast<int64_t>(b) * N + e] = run;
            run += c;
        }
        tot[e] = run;
    }
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    // exclusive scan of tot[0..N) in chunks of SCAN_THREADS
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base_e = 0; base_e < N; base_e += SCAN_THREADS) {
        const int e = base_e + threadIdx.x;
        const int v = (e < N) ? tot[e] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        if (lane == 31) warp_sums[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int ws = warp_sums[lane];
            int wi = ws;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += u;
            }
            warp_sums[lane] = wi - ws;  // exclusive prefix of warp totals
        }
        __syncthreads();
        const int excl = carry + warp_sums[warp] + incl - v;
        if (e < N) offsets[e] = excl;
        __syncthreads();
        if (threadIdx.x == SCAN_THREADS - 1) carry = excl + v;
        __syncthreads();
    }
    if (threadIdx.x == 0) offsets[N] = carry;
}

__global__ void __launch_bounds__(PB)
    perm_scatter_kernel(const int32_t* __restrict__ idx, int T, int K, int N, int E,
                        const int32_t* __restrict__ base, const int32_t* __restrict__ offsets,
                        int32_t* __restrict__ row_token, int32_t* __restrict__ pair_row) {
    extern __shared__ uint32_t mask[];
    for (int i = threadIdx.x; i < N * MASK_WORDS; i += PB) mask[i] = 0;
    __syncthreads();
    build_masks(idx, T, K, N, E, mask, nullptr);
    __syncthreads();
    const int t = blockIdx.x * PB + threadIdx.x;
    if (t >= T) return;
    const int w = threadIdx.x >> 5;
    const uint32_t below = (1u << (threadIdx.x & 31)) - 1u;
    for (int r = 0; r < K; ++r) {
        const int e = idx[static_cast<int64_t>(t) * K + r];
        int row = -1;
        if (e >= 0 && e < N) {
            int rank = __popc(mask[e * MASK_WORDS + w] & below);
            for (int j = 0; j < w; ++j) rank += __popc(mask[e * MASK_WORDS + j]);
            row = offsets[e] + base[static_cast<int64_t>(blockIdx.x) * N + e] + rank;
            row_token[row] = t;
        }
        pair_row[static_cast<int64_t>(t) * K + r] = row;
    }
}

// All of it in one block when the batch is one block of tokens (T <= 256, decode-sized batches):
// masks and counts as in perm_count_kernel, the exclusive scan of the counts over the experts in
// shared memory, and the scatter of perm_scatter_kernel with every base 0; one launch instead of
// three.
__global__ void __launch_bounds__(PB)
    perm_single_kernel(const int32_t* __restrict__ idx, int T, int K, int N, int E,
                       int32_t* __restrict__ offsets, int32_t* __restrict__ row_token,
                       int32_t* __restrict__ pair_row, uint32_t* __restrict__ status) {
    extern __shared__ uint32_t mask[];              // [N][MASK_WORDS]
    int32_t* offs = reinterpret_cast<int32_t*>(mask + N * MASK_WORDS);  // [N]
    __shared__ int32_t warp_sums[PB / 32];
    __shared__ int32_t carry;
    for (int i = threadIdx.x; i < N * MASK_WORDS; i += PB) mask[i] = 0;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const bool bad = build_masks(idx, T, K, N, E, mask, status);
    if (__syncthreads_or(bad) && threadIdx.x == 0) set_status(status, LC_MOE_DEV_IDX_RANGE);
    // exclusive scan of the per-expert counts, PB experts at a time
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int e0 = 0; e0 < N; e0 += PB) {
        const int e = e0 + threadIdx.x;
        int v = 0;
        if (e < N) {
#pragma unroll
            for (int w = 0; w < MASK_WORDS; ++w) v += __popc(mask[e * MASK_WORDS + w]);
        }
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        if (lane == 31) warp_sums[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int ws = lane < PB / 32 ? warp_sums[lane] : 0;
            int wi = ws;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += u;
            }
            if (lane < PB / 32) warp_sums[lane] = wi - ws;  // exclusive prefix of warp totals
        }
        __syncthreads();
        const int excl = carry + warp_sums[warp] + incl - v;
        if (e < N) {
            offs[e] = excl;
            offsets[e] = excl;
        }
        __syncthreads();
        if (threadIdx.x == PB - 1) carry = excl + v;
        __syncthreads();
    }
    if (threadIdx.x == 0) offsets[N] = carry;
    const int t = threadIdx.x;
    if (t >= T) return;
    const int w = threadIdx.x >> 5;
    const uint32_t below = (1u << (threadIdx.x & 31)) - 1u;
    for (int r = 0; r < K; ++r) {
        const int e = idx[static_cast<int64_t>(t) * K + r];
        int row = -1;
        if (e >= 0 && e < N) {
            int rank = __popc(mask[e * MASK_WORDS + w] & below);
            for (int j = 0; j < w; ++j) rank += __popc(mask[e * MASK_WORDS + j]);
            row = offs[e] + rank;
            row_token[row] = t;
        }
        pair_row[static_cast<int64_t>(t) * K + r] = row;
    }
}

constexpr int GATHER_THREADS = 256;

__global__ void __launch_bounds__(GATHER_THREADS)
    gather_kernel(const uint4* __restrict__ x, int T, int d8, int K, const int32_t* __restrict__ pair_row,
                  uint4* __restrict__ x_perm, const float* __restrict__ sx, float* __restrict__ s_row) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (GATHER_THREADS / 32);
    for (int t = blockIdx.x * (GATHER_THREADS / 32) + warp; t < T; t += warps_total) {
        const int my_row = (lane < K) ? pair_row[static_cast<int64_t>(t) * K + lane] : -1;
        const uint32_t dests = __ballot_sync(0xffffffffu, my_row >= 0);
        if (!dests) continue;
        if (s_row && my_row >= 0) s_row[my_row] = sx[t];  // row scale of E4M3 rows
        const uint4* src = x + static_cast<int64_t>(t) * d8;
        for (int c0 = 0; c0 < d8; c0 += 128) {  // warp-uniform trip count; 4 loads in flight
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c0 + 32 * u + lane;
                v[u] = c < d8 ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
            }
            uint32_t m = dests;
            while (m) {
                const int r = __ffs(m) - 1;
                m &= m - 1;
                const int row = __shfl_sync(0xffffffffu, my_row, r);
                uint4* dst = x_perm + static_cast<int64_t>(row) * d8;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int c = c0 + 32 * u + lane;
                    if (c < d8) dst[c] = v[u];
                }
            }
        }
    }
}

// Row gather with bulk async copies: warp w of a block owns two shared-memory row slots. Its
// first lane loads token t's row with one cp.async.bulk (completion on the slot's mbarrier), and
// once it has landed writes it to each of the token's FFN rows with one bulk store per row; the
// next token's row is loaded into the other slot meanwhile, after the stores that last read
// that slot are done reading it. The copies never pass through registers. Every wait is bounded
// (LC_MOE_DEV_WAIT_TIMEOUT).
constexpr int GB_WARPS = 4;
constexpr uint32_t GB_MAX_ROW_BYTES = 25600;  // 2 slots x 4 warps within 200 KB of shared memory

__global__ void __launch_bounds__(GB_WARPS * 32)
    gather_bulk_kernel(const uint8_t* __restrict__ x, int T, uint32_t row_bytes, int K,
                       const int32_t* __restrict__ pair_row, uint8_t* __restrict__ x_perm,
                       const float* __restrict__ sx, float* __restrict__ s_row, uint32_t* status,
                       uint64_t wait_ns) {
    extern __shared__ __align__(128) uint8_t gsm[];
    __shared__ uint64_t bars[GB_WARPS][2];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* slot0 = gsm + static_cast<size_t>(2 * warp) * row_bytes;
    uint8_t* slot1 = slot0 + row_bytes;
    if (lane == 0) {
        mbar_init(&bars[warp][0], 1);
        mbar_init(&bars[warp][1], 1);
        fence_mbar_init();
    }
    __syncwarp();
    const int stride = gridDim.x * GB_WARPS;
    int t = blockIdx.x * GB_WARPS + warp;
    uint32_t ph0 = 0, ph1 = 0;
    int b = 0;
    if (lane == 0 && t < T) {
        mbar_arrive_expect_tx(&bars[warp][0], row_bytes);
        bulk_load_g2s(slot0, x + static_cast<int64_t>(t) * row_bytes, row_bytes, &bars[warp][0]);
    }
    for (; t < T; t += stride) {
        const int tn = t + stride;
        const int my_row = (lane < K) ? pair_row[static_cast<int64_t>(t) * K + lane] : -1;
        if (s_row && my_row >= 0) s_row[my_row] = sx[t];  // row scale of E4M3 rows
        const uint32_t dests = __ballot_sync(0xffffffffu, my_row >= 0);
        uint8_t* cur = b ? slot1 : slot0;
        uint8_t* nxt = b ? slot0 : slot1;
        int got = 1;
        if (lane == 0) {
            const bool nxt_issued = tn < T;
            if (nxt_issued) {
                // the stores issued from the other slot (previous token) must be done reading it
                bulk_wait_read<0>();
                mbar_arrive_expect_tx(&bars[warp][b ^ 1], row_bytes);
                bulk_load_g2s(nxt, x + static_cast<int64_t>(tn) * row_bytes, row_bytes, &bars[warp][b ^ 1]);
            }
            const uint32_t ph = b ? ph1 : ph0;
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&bars[warp][b], ph)) {
                if (globaltimer_ns() - t0 > wait_ns) {
                    set_status(status, LC_MOE_DEV_WAIT_TIMEOUT);
                    got = 0;
                    break;
                }
            }
            if (got) {
                fence_proxy_async_smem();
            } else if (nxt_issued) {
                // do not leave while the other slot's load may still be writing it
                const uint32_t phn = b ? ph0 : ph1;
                const uint64_t t1 = globaltimer_ns();
                while (!mbar_try_wait(&bars[warp][b ^ 1], phn) && globaltimer_ns() - t1 < wait_ns) {
                }
            }
        }
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) break;
        if (b) ph1 ^= 1u;
        else ph0 ^= 1u;
        uint32_t m = dests;
        while (m) {
            const int r = __ffs(m) - 1;
            m &= m - 1;
            const int row = __shfl_sync(0xffffffffu, my_row, r);
            if (lane == 0) bulk_store_s2g(x_perm + static_cast<int64_t>(row) * row_bytes, cur, row_bytes);
        }
        if (lane == 0) bulk_commit();
        b ^= 1;
    }
    if (lane == 0) bulk_wait<0>();  // the last stores have left shared memory and landed
}

cudaError_t launch_gather_rows(const void* x, int T, uint32_t row_bytes, int K, const int32_t* pair_row,
                               void* x_perm, const float* sx, float* s_row, uint32_t* status,
                               cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    if (T == 0) return cudaSuccess;
    if (row_bytes <= GB_MAX_ROW_BYTES) {
        const size_t smem = static_cast<size_t>(2 * GB_WARPS) * row_bytes;
        static PerDeviceOnce setup;
        const cudaError_t e = setup.run([](int) {
            return cudaFuncSetAttribute(gather_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(2 * GB_WARPS * GB_MAX_ROW_BYTES));
        });
        if (e != cudaSuccess) return e;
        int blocks = (T + GB_WARPS - 1) / GB_WARPS;
        const int per_sm = smem ? static_cast<int>((200u * 1024u) / smem) : 8;
        const int cap = di->sm_count * (per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm));
        if (blocks > cap) blocks = cap;
        gather_bulk_kernel<<<blocks, GB_WARPS * 32, smem, st>>>(static_cast<const uint8_t*>(x), T, row_bytes, K,
                                                                 pair_row, static_cast<uint8_t*>(x_perm), sx,
                                                                 s_row, status, wait_limit_ns());
        return cudaGetLastError();
    }
    const int warps = GATHER_THREADS / 32;
    int blocks = (T + warps - 1) / warps;
    if (blocks > di->sm_count * 8) blocks = di->sm_count * 8;
    gather_kernel<<<blocks, GATHER_THREADS, 0, st>>>(static_cast<const uint4*>(x), T, static_cast<int>(row_bytes / 16),
                                                      K, pair_row, static_cast<uint4*>(x_perm), sx, s_row);
    return cudaGetLastError();
}

}  // namespace

size_t permute_scratch_bytes(int T, int N) {
    const size_t nblk = (static_cast<size_t>(T) + PB - 1) / PB;
    return 2 * nblk * static_cast<size_t>(N) * sizeof(int32_t);
}

cudaError_t launch_permute(const int32_t* idx, int T, int K, int N, int E, int32_t* offsets,
                           int32_t* row_token, int32_t* pair_row, int32_t* scratch,
                           uint32_t* status, cudaStream_t st) {
    const int nblk = (T + PB - 1) / PB;
    int32_t* cnt = scratch;
    int32_t* base = scratch + static_cast<size_t>(nblk) * N;
    const size_t mask_bytes = static_cast<size_t>(N) * MASK_WORDS * sizeof(uint32_t);
    static PerDeviceOnce setup;
    cudaError_t e = setup.run([](int) {
        // masks of up to 2048 experts take 64 KB of shared memory (plus their offsets: 72 KB)
        cudaError_t r = cudaFuncSetAttribute(perm_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             2048 * MASK_WORDS * 4);
        if (r != cudaSuccess) return r;
        r = cudaFuncSetAttribute(perm_single_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 2048 * (MASK_WORDS + 1) * 4);
        if (r != cudaSuccess) return r;
        return cudaFuncSetAttribute(perm_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    2048 * MASK_WORDS * 4);
    });
    if (e != cudaSuccess) return e;
    if (nblk <= 1) {
        perm_single_kernel<<<1, PB, static_cast<size_t>(N) * (MASK_WORDS + 1) * sizeof(uint32_t), st>>>(
            idx, T, K, N, E, offsets, row_token, pair_row, status);
        return cudaGetLastError();
    }
    if (nblk > 0) {
        perm_count_kernel<<<nblk, PB, mask_bytes, st>>>(idx, T, K, N, E, cnt, status);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    perm_scan_kernel<<<1, SCAN_THREADS, static_cast<size_t>(N) * sizeof(int32_t), st>>>(cnt, nblk, N, base, offsets);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (nblk > 0) {
        perm_scatter_kernel<<<nblk, PB, mask_bytes, st>>>(idx, T, K, N, E, base, offsets, row_token, pair_row);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_gather(const void* x, int T, int d, int K, const int32_t* pair_row, void* x_perm,
                          uint32_t* status, cudaStream_t st) {
    return launch_gather_rows(x, T, static_cast<uint32_t>(d) * 2, K, pair_row, x_perm, nullptr, nullptr,
                              status, st);
}

cudaError_t launch_gather_e4m3(const void* xq, const float* sx, int T, int d, int K,
                               const int32_t* pair_row, void* x_perm, float* s_row, uint32_t* status,
                               cudaStream_t st) {
    return launch_gather_rows(xq, T, static_cast<uint32_t>(d), K, pair_row, x_perm, sx, s_row, status, st);
}

// ---------------------------------------------------------------------------------------------
// Allocation-free grouping: the same three kernels, with the two grouping tables in a file-scope
// device array instead of a caller-provided workspace, for callers that cannot allocate device
// memory. Capacity: ceil(T/256) * N <= kNoAllocTableEntries (for example T <= 65536 tokens with
// N = 512 experts, or T <= 16384 with N = 2048). Every call on a device shares this one array, so
// calls that overlap on the GPU race on it; calls ordered on one stream do not. Both tables are
// fully rewritten by every call (counts by the count kernel, bases by the scan kernel), so nothing
// left over from an earlier call is read.
// ---------------------------------------------------------------------------------------------

namespace {

constexpr int64_t kNoAllocTableEntries = 131072;  // per table: 512 KB of int32
__device__ __align__(256) int32_t g_noalloc_tables[2 * kNoAllocTableEntries];

// Device address of g_noalloc_tables on the current device. In host code the symbol is only a
// stand-in for the device array; kernels must get this address. The lookup runs on a device's
// first call and is kept once it succeeds; a failed lookup (for example one attempted inside a
// stream capture) is returned and tried again on the next call.
cudaError_t noalloc_tables_ptr(int32_t** out) {
    static PerDeviceOnce lookup;
    static int32_t* ptrs[PerDeviceOnce::kMaxDevices];
    cudaError_t e = lookup.run([](int dev) {
        void* p = nullptr;
        const cudaError_t r = cudaGetSymbolAddress(&p, g_noalloc_tables);
        if (r == cudaSuccess) ptrs[dev] = static_cast<int32_t*>(p);
        return r;
    });
    if (e != cudaSuccess) return e;
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    *out = ptrs[dev];
    return cudaSuccess;
}

}  // namespace

bool permute_noalloc_fits(int T, int N) {
    const int64_t nblk = (static_cast<int64_t>(T) + PB - 1) / PB;
    return nblk * N <= kNoAllocTableEntries;
}

cudaError_t launch_permute_noalloc(const int32_t* idx, int T, int K, int N, int E, int32_t* offsets,
                                   int32_t* row_token, int32_t* pair_row, uint32_t* status,
                                   cudaStream_t st) {
    if (!permute_noalloc_fits(T, N)) return cudaErrorInvalidValue;
    int32_t* tables = nullptr;
    cudaError_t e = noalloc_tables_ptr(&tables);
    if (e != cudaSuccess) return e;
    // launch_permute lays out the count table first and the base table after it, each
    // ceil(T/256) * N entries: both fit in the array by the capacity check above.
    return launch_permute(idx, T, K, N, E, offsets, row_token, pair_row, tables, status, st);
}

}  // namespace lcmoe
