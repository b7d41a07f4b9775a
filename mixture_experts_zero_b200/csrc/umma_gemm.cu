// umma_gemm.cu -- the router GEMM on the sm_100a tensor cores:
//
//   logits[T, E] (fp32) = x[T, d] * Wr[E, d]^T
//
// over all N + Z experts (the router of the LongCat-Flash llm-wiki entity page, section 2.1, picks
// among FFN and zero-computation experts alike). fp32 logits feed the softmax / top-K kernel.
//
// One persistent, warp-specialised kernel (one CTA of 256 threads per SM):
//   warp 0 (one lane)  TMA producer: 128 x 64 tiles of x and BN x 64 tiles of Wr, 128-byte
//                      swizzle, into a 4-stage shared-memory ring (full/empty mbarriers);
//   warp 1 (one lane)  tcgen05.mma.cta_group::1.kind::f16 128 x BN x 16 with fp32 accumulators in
//                      TMEM, two 256-column buffers so the epilogue of one tile overlaps the main
//                      loop of the next; tcgen05.commit releases smem stages;
//   warp 1 (all)       TMEM allocation / deallocation (512 columns);
//   warps 4..7         epilogue: tcgen05.ld (one TMEM lane = one token row), fp32 stores.
// Tile t (128 tokens x BN experts) goes to CTA t mod gridDim. Rows past T and experts past E are
// read as zero by TMA and never stored. Every wait is bounded (lc_moe_set_wait_limit_ns); a wait
// that runs out raises a CTA-wide abort, records LC_MOE_DEV_WAIT_TIMEOUT, drains its in-flight
// copies and MMAs, and frees TMEM.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace lcmoe {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;                      // 64 bf16 = 128 bytes = one swizzle row
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;        // 16 KB
constexpr int B_BYTES_MAX = 256 * BK * 2;   // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES_MAX;
constexpr int TMEM_COLS = 512;              // two 128 x 256 fp32 accumulators
constexpr int NUM_THREADS = 256;

struct RouterArgs {
    float* out;              // [rows, ldo]
    uint32_t* status;
    uint64_t wait_ns;
    int64_t ldo;             // output row stride in elements (E)
    int rows;                // T
    int kdim;                // d (multiple of 64)
    int n_out;               // E
    int bn;                  // MMA N (tile width)
    int ntiles;              // tiles along the experts
};

struct SmemLayout {
    static constexpr int bars_off = STAGES * STAGE_BYTES;
    static constexpr int n_bars = 2 * STAGES + 5;  // full, empty, tfull[2], tempty[2], drain
    static constexpr int misc_off = bars_off + n_bars * 8;
    static constexpr size_t bytes() { return 1024 + misc_off + 16; }
};

__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    router_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                       const RouterArgs g) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + SmemLayout::bars_off);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SmemLayout::misc_off);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SmemLayout::misc_off + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&mapA);
        tma_prefetch_desc(&mapB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int total = ((g.rows + BM - 1) / BM) * g.ntiles;
    const int nk = g.kdim / BK;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------------ TMA producer --
        const uint32_t tx_bytes = static_cast<uint32_t>(A_BYTES + g.bn * BK * 2);
        int s = 0;
        uint32_t ph = 0;
        int issued = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            const int mt = tile / g.ntiles;
            const int n0 = (tile - mt * g.ntiles) * g.bn;
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait(&empty[s], ph ^ 1u, g.wait_ns, abort_flag, g.status)) {
                    ok = false;
                    break;
                }
                uint8_t* sa = smem + s * STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], tx_bytes);
                tma_load_2d(sa, &mapA, &full[s], kb * BK, mt * BM);
                tma_load_2d(sa + A_BYTES, &mapB, &full[s], kb * BK, n0);
                ++issued;
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        if (!ok) {
            // wait (bounded) for the copies that may still be landing in shared memory
            for (int i = 0; i < STAGES && i < issued; ++i) {
                if (s == 0) {
                    s = STAGES - 1;
                    ph ^= 1u;
                } else {
                    --s;
                }
                mbar_wait_drain(&full[s], ph, g.wait_ns);
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------------- MMA issuer --
        const uint32_t idesc = idesc_bf16_f32(BM, g.bn);
        int s = 0;
        uint32_t ph = 0;
        int acc = 0;
        uint32_t aph = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            if (!mbar_wait(&tempty[acc], aph ^ 1u, g.wait_ns, abort_flag, g.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait(&full[s], ph, g.wait_ns, abort_flag, g.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t* sa = smem + s * STAGE_BYTES;
                const uint64_t ad = sw128_kmajor_desc(smem_u32(sa));
                const uint64_t bd = sw128_kmajor_desc(smem_u32(sa + A_BYTES));
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    // +32 bytes along K inside the 128-byte swizzle row = +2 in the address field
                    umma_bf16(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
                }
                umma_commit(&empty[s]);
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (!ok) break;
            umma_commit(&tfull[acc]);
            acc ^= 1;
            if (acc == 0) aph ^= 1u;
        }
        umma_commit(drain);
        mbar_wait_drain(drain, 0, g.wait_ns);
    } else if (warp >= 4) {
        // --------------------------------------------------------------------- epilogue --
        const int q = warp - 4;  // TMEM lane quarter this warp may read
        int acc = 0;
        uint32_t aph = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const int mt = tile / g.ntiles;
            const int n0 = (tile - mt * g.ntiles) * g.bn;
            if (!mbar_wait(&tfull[acc], aph, g.wait_ns, abort_flag, g.status)) break;
            tc_fence_after();
            const int r = mt * BM + q * 32 + lane;
            const bool valid = r < g.rows;
            const uint32_t tb =
                tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * 256);
            for (int c = 0; c < g.bn; c += 32) {
                const int col0 = n0 + c;
                if (col0 >= g.n_out) break;  // warp-uniform
                uint32_t v[32];
                tmem_ld_32x32b_x32(tb + c, v);
                tmem_ld_wait();
                if (valid) {
                    float* dst = g.out + static_cast<int64_t>(r) * g.ldo + col0;
                    if (col0 + 32 <= g.n_out && (g.ldo & 3) == 0) {
                        float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            d4[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (col0 + j < g.n_out) dst[j] = __uint_as_float(v[j]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) aph ^= 1u;
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

}  // namespace

// Row-major bf16 matrix [rows, cols] read in boxes of box_rows x 64 with the 128-byte swizzle.
bool make_tma_map_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tma_map_2d_u8(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_router_gemm(const void* x, const void* wr, float* logits, int T, int d, int E,
                               uint32_t* status, cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    const int bn_max = ((E + 31) / 32) * 32 < 256 ? ((E + 31) / 32) * 32 : 256;
    int bn = bn_max;
    const int m_tiles = (T + BM - 1) / BM;
    const int sms = di->sm_count;
    if (m_tiles * ((E + bn - 1) / bn) < sms) {
        // few token tiles (decode-sized T): narrower expert tiles, down to 32, so that more SMs
        // stream the router weight
        while (bn > 32 && m_tiles * ((E + bn - 1) / bn) < sms) bn = ((bn / 2 + 31) / 32) * 32;
    } else {
        // at least one full wave: the width from bn_max down to 128 (multiples of 32) with the
        // least waves x width, i.e. the last wave filled best (a tile's time grows with its width);
        // ties keep the wider tile
        int64_t best = -1;
        for (int c = bn_max; c >= 128 || c == bn_max; c -= 32) {
            const int64_t tiles = static_cast<int64_t>(m_tiles) * ((E + c - 1) / c);
            const int64_t cost = ((tiles + sms - 1) / sms) * c;
            if (best < 0 || cost < best) {
                best = cost;
                bn = c;
            }
            if (c <= 32) break;
        }
    }
    CUtensorMap ma, mb;
    if (!make_tma_map_2d(&ma, x, static_cast<uint64_t>(T), d, BM)) return cudaErrorInvalidValue;
    if (!make_tma_map_2d(&mb, wr, static_cast<uint64_t>(E), d, bn)) return cudaErrorInvalidValue;
    RouterArgs a{};
    a.out = logits;
    a.status = status;
    a.wait_ns = wait_limit_ns();
    a.ldo = E;
    a.rows = T;
    a.kdim = d;
    a.n_out = E;
    a.bn = bn;
    a.ntiles = (E + bn - 1) / bn;
    const int tiles = ((T + BM - 1) / BM) * a.ntiles;
    const int grid = tiles < di->sm_count ? tiles : di->sm_count;
    const size_t smem = SmemLayout::bytes();
    static PerDeviceOnce setup;
    const cudaError_t e = setup.run([smem](int) {
        return cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem));
    });
    if (e != cudaSuccess) return e;
    router_gemm_kernel<<<grid, NUM_THREADS, smem, st>>>(ma, mb, a);
    return cudaGetLastError();
}

}  // namespace lcmoe
