// umma_gemm.cu -- the dense contractions of the MoE layer on the sm_100a tensor cores.
//
//   router GEMM : logits[T, E] (fp32)  = x[T, d] * Wr[E, d]^T
//   grouped GEMM 1 (per FFN expert e, over the rows routed to e):
//                 H[rows_e, I] (bf16) = silu(X_e Wg[e]^T) * (X_e Wu[e]^T)   (SwiGLU in the epilogue)
//   grouped GEMM 2: Y[rows_e, d] (bf16) = H_e Wd[e]^T
//
// The FFN experts are the N "standard FFN experts" of the MoE equation (LongCat-Flash llm-wiki
// entity page, section 2.1); only rows routed to FFN experts reach these GEMMs, so the Z
// zero-computation experts cost no FLOPs here. Expert width I comes from the section 1 table.
//
// One persistent, warp-specialised kernel per GEMM (one CTA of 256 threads per SM):
//   warp 0 (one lane)  TMA producer into a 4-stage shared-memory ring (128-byte swizzle,
//                      full/empty mbarriers);
//   warp 1 (one lane)  tcgen05.mma issuer, fp32 accumulators in TMEM, two 256-column buffers so
//                      the epilogue of one tile overlaps the main loop of the next;
//   warp 1 (all)       TMEM allocation / deallocation (512 columns);
//   warps 4..7         epilogue: tcgen05.ld of the accumulator, SwiGLU / conversion, stores.
//
// Tiles of the grouped GEMMs come in two kinds, chosen per expert from its row count c_e:
//   row tiles (c_e >= 128): 128 rows of the expert x 256 accumulator columns. A = the expert's
//     rows, B = weight rows. GEMM 1 loads 128 gate rows and the matching 128 up rows as B, so the
//     accumulator holds gate and up side by side for each row. Rows past c_e in the last tile are
//     computed and not stored.
//   weight tiles (0 < c_e < 128, "swap"): 128 weight rows x round_up(c_e, 32) accumulator columns.
//     A = weight rows, B = the expert's rows, so a lightly used expert costs one pass over its
//     weights and no 128-row padding. GEMM 1 issues two MMAs per k-step on the same B: 128 gate
//     rows into accumulator columns [0, 128) and the matching 128 up rows into [128, 256), so one
//     TMEM lane holds both the gate and the up value of its feature for every row.
// The tile list is built on the device from offsets[N+1]: per-expert tile counts of each kind are
// prefix-summed in shared memory by every CTA; the list is every row tile in expert order, then
// every weight tile. Tile t goes to CTA t mod gridDim; there is no host synchronisation between
// grouping and GEMMs. Consecutive row tiles of a hot expert share its weight tiles through L2;
// merging the two kinds in proportion (to overlap HBM-bound weight tiles with compute-bound row
// tiles) spread those row tiles out in time and raised the grouped GEMM 1's DRAM reads from 31.9 to
// 51.6 GB at the prefill workload, so the kinds run one after the other. Weight-tile loads carry an
// L2 evict-first hint (each such weight byte is used once).
// Every wait is bounded (lc_moe_set_wait_limit_ns); a wait that runs out raises a CTA-wide abort,
// records LC_MOE_DEV_WAIT_TIMEOUT, drains its in-flight copies and MMAs, and frees TMEM.
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
constexpr int SWAP_BOX = 32;                // token rows per TMA box of a weight tile
constexpr int COLD_ROWS = 128;              // experts with fewer rows use weight tiles

enum Mode : int { MODE_ROUTER = 0, MODE_SWIGLU = 1, MODE_DOWN = 2 };

struct GemmArgs {
    const int32_t* offsets;  // grouped: [n_groups + 1] row offsets
    void* out;               // router: fp32 [rows, ldo]; grouped: bf16 [rows_cap, ldo]
    uint32_t* status;
    uint64_t wait_ns;
    int64_t rows_cap;        // rows of the row-operand buffers (and of the output) that exist
    int64_t ldo;             // output row stride in elements
    int n_groups;            // grouped: N; router: 1
    int rows;                // router: T
    int kdim;                // reduction length (multiple of 64)
    int n_out;               // output columns
    int bn;                  // MMA N of a row tile
    int tile_cols;           // output columns per row tile
    int ntiles;              // row tiles along the output columns
    int b_group_rows;        // rows of the weight matrix per group
    int up_off;              // SwiGLU: row offset of Wu inside a group (= I)
    int s_cols;              // output columns per weight tile (0: no weight tiles)
    int s_tiles;             // weight tiles per cold expert
};

struct SmemLayout {
    static constexpr int bars_off = STAGES * STAGE_BYTES;
    // full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
    static constexpr int n_bars = 2 * STAGES + 5;
    static constexpr int misc_off = bars_off + n_bars * 8;     // tmem slot, abort flag
    static constexpr int table_off = (misc_off + 16 + 15) & ~15;
    static size_t bytes(int n_groups) {
        return 1024 + table_off + 3 * static_cast<size_t>(n_groups + 1) * 4;
    }
};

struct Tile {
    int swap;       // 0: row tile, 1: weight tile
    int grp;
    int64_t row0;   // first row of the row operand
    int rows;       // valid rows from row0
    int n0;         // first output column
    int ntok;       // weight tile: MMA N (rows rounded up to SWAP_BOX)
};

// Bounded wait used while draining after an abort: ignores the abort flag.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
    return g / (1.0f + __expf(-g)) * u;
}

// largest e in [0, n - 1] with pre[e] <= v (pre non-decreasing, pre[0] = 0 <= v)
__device__ __forceinline__ int upper_group(const int32_t* pre, int n, int v) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= v) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                     const __grid_constant__ CUtensorMap mapSA, const __grid_constant__ CUtensorMap mapSB,
                     const GemmArgs g) {
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
    int32_t* offs_s = reinterpret_cast<int32_t*>(smem + SmemLayout::table_off);
    int32_t* rpre_s = offs_s + (g.n_groups + 1);  // first row tile of each group
    int32_t* spre_s = rpre_s + (g.n_groups + 1);  // first weight tile of each group

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    constexpr bool GROUPED = MODE != MODE_ROUTER;

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
        if (GROUPED && g.s_cols > 0) {
            tma_prefetch_desc(&mapSA);
            tma_prefetch_desc(&mapSB);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    if (GROUPED) {
        for (int e = threadIdx.x; e <= g.n_groups; e += NUM_THREADS) offs_s[e] = g.offsets[e];
    }
    __syncthreads();
    if (GROUPED && warp == 2) {
        // per-group tile counts of each kind, exclusive prefix sums
        int run_r = 0, run_s = 0;
        if (lane == 0) {
            rpre_s[0] = 0;
            spre_s[0] = 0;
        }
        for (int base = 0; base < g.n_groups; base += 32) {
            const int e = base + lane;
            int nr = 0, ns = 0;
            if (e < g.n_groups) {
                int cnt = offs_s[e + 1] - offs_s[e];
                if (cnt < 0) {
                    cnt = 0;
                    set_status(g.status, LC_MOE_DEV_IDX_RANGE);
                }
                if (g.s_cols > 0 && cnt > 0 && cnt < COLD_ROWS) ns = g.s_tiles;
                else nr = (cnt + BM - 1) / BM * g.ntiles;
            }
            int ir = nr, is = ns;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int vr = __shfl_up_sync(0xffffffffu, ir, o);
                const int vs = __shfl_up_sync(0xffffffffu, is, o);
                if (lane >= o) {
                    ir += vr;
                    is += vs;
                }
            }
            if (e < g.n_groups) {
                rpre_s[e + 1] = run_r + ir;
                spre_s[e + 1] = run_s + is;
            }
            run_r += __shfl_sync(0xffffffffu, ir, 31);
            run_s += __shfl_sync(0xffffffffu, is, 31);
        }
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int total_r = GROUPED ? rpre_s[g.n_groups] : ((g.rows + BM - 1) / BM) * g.ntiles;
    const int total_s = GROUPED ? spre_s[g.n_groups] : 0;
    const int total = total_r + total_s;
    const int nk = g.kdim / BK;

    auto decode = [&](int tile) {
        Tile tl;
        int idx = tile;
        tl.swap = 0;
        if (total_s > 0) {
            // all row tiles (in expert order), then all weight tiles
            tl.swap = tile >= total_r;
            idx = tl.swap ? tile - total_r : tile;
        }
        if (!GROUPED) {
            const int mt = idx / g.ntiles;
            tl.grp = 0;
            tl.row0 = static_cast<int64_t>(mt) * BM;
            tl.rows = min(BM, g.rows - mt * BM);
            tl.n0 = (idx - mt * g.ntiles) * g.tile_cols;
            tl.ntok = 0;
        } else if (!tl.swap) {
            const int e = upper_group(rpre_s, g.n_groups, idx);
            const int local = idx - rpre_s[e];
            const int mt = local / g.ntiles;
            tl.grp = e;
            tl.row0 = static_cast<int64_t>(offs_s[e]) + static_cast<int64_t>(mt) * BM;
            tl.rows = min(BM, offs_s[e + 1] - offs_s[e] - mt * BM);
            tl.n0 = (local - mt * g.ntiles) * g.tile_cols;
            tl.ntok = 0;
        } else {
            const int e = upper_group(spre_s, g.n_groups, idx);
            tl.grp = e;
            tl.row0 = offs_s[e];
            tl.rows = offs_s[e + 1] - offs_s[e];
            tl.n0 = (idx - spre_s[e]) * g.s_cols;
            tl.ntok = (tl.rows + SWAP_BOX - 1) / SWAP_BOX * SWAP_BOX;
        }
        return tl;
    };

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------------ TMA producer --
        const uint64_t pol_stream = l2_policy_evict_first();
        const uint64_t pol_normal = l2_policy_evict_normal();
        int s = 0;
        uint32_t ph = 0;
        int issued = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            const Tile tl = decode(tile);
            const uint32_t tx_bytes = static_cast<uint32_t>(
                tl.swap ? (MODE == MODE_SWIGLU ? 2 : 1) * A_BYTES + tl.ntok * BK * 2
                        : A_BYTES + g.bn * BK * 2);
            const int wrow = (MODE == MODE_ROUTER) ? tl.n0 : tl.grp * g.b_group_rows + tl.n0;
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait(&empty[s], ph ^ 1u, g.wait_ns, abort_flag, g.status)) {
                    ok = false;
                    break;
                }
                uint8_t* sa = smem + s * STAGE_BYTES;
                uint8_t* sb = sa + A_BYTES;
                mbar_arrive_expect_tx(&full[s], tx_bytes);
                if (!tl.swap) {
                    tma_load_2d_hint(sa, &mapA, &full[s], kb * BK, static_cast<int32_t>(tl.row0), pol_normal);
                    if (MODE == MODE_SWIGLU) {
                        const int half = g.bn / 2;
                        tma_load_2d_hint(sb, &mapB, &full[s], kb * BK, wrow, pol_normal);
                        tma_load_2d_hint(sb + half * 128, &mapB, &full[s], kb * BK, wrow + g.up_off, pol_normal);
                    } else {
                        tma_load_2d_hint(sb, &mapB, &full[s], kb * BK, wrow, pol_normal);
                    }
                } else {
                    // weight rows into A (GEMM 1: gate rows into A, up rows into the first half of
                    // the B slot), the expert's rows after them
                    tma_load_2d_hint(sa, &mapSA, &full[s], kb * BK, wrow, pol_stream);
                    uint8_t* st = sb;
                    if (MODE == MODE_SWIGLU) {
                        tma_load_2d_hint(sb, &mapSA, &full[s], kb * BK, wrow + g.up_off, pol_stream);
                        st = sb + A_BYTES;
                    }
                    for (int b = 0; b < tl.ntok; b += SWAP_BOX)
                        tma_load_2d_hint(st + b * 128, &mapSB, &full[s], kb * BK,
                                         static_cast<int32_t>(tl.row0 + b), pol_normal);
                }
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
        int s = 0;
        uint32_t ph = 0;
        int acc = 0;
        uint32_t aph = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            const Tile tl = decode(tile);
            const uint32_t idesc = idesc_bf16_f32(BM, tl.swap ? tl.ntok : g.bn);
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
                if (MODE == MODE_SWIGLU && tl.swap) {
                    // gate rows (A slot) and up rows (first half of the B slot) times the rows
                    const uint64_t td = sw128_kmajor_desc(smem_u32(sa + 2 * A_BYTES));
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        umma_bf16(d_tmem, ad + 2 * kk, td + 2 * kk, idesc, (kb | kk) != 0);
                        umma_bf16(d_tmem + 128, bd + 2 * kk, td + 2 * kk, idesc, (kb | kk) != 0);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // +32 bytes along K inside the 128-byte swizzle row = +2 in the address field
                        umma_bf16(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
                    }
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
            const Tile tl = decode(tile);
            if (!mbar_wait(&tfull[acc], aph, g.wait_ns, abort_flag, g.status)) break;
            tc_fence_after();
            const uint32_t tb =
                tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * 256);
            if (!tl.swap) {
                // one TMEM lane = one output row
                const int r = q * 32 + lane;
                const int64_t grow = tl.row0 + r;
                const bool valid = r < tl.rows && grow >= 0 && grow < g.rows_cap;
                if (MODE == MODE_ROUTER) {
                    float* out = static_cast<float*>(g.out);
                    for (int c = 0; c < g.bn; c += 32) {
                        const int col0 = tl.n0 + c;
                        if (col0 >= g.n_out) break;  // warp-uniform
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(tb + c, v);
                        tmem_ld_wait();
                        if (valid) {
                            float* dst = out + grow * g.ldo + col0;
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
                } else if (MODE == MODE_SWIGLU) {
                    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out);
                    const int half = g.bn / 2;
                    for (int c = 0; c < half; c += 32) {
                        uint32_t gv[32], uv[32];
                        tmem_ld_32x32b_x32(tb + c, gv);
                        tmem_ld_32x32b_x32(tb + half + c, uv);
                        tmem_ld_wait();
                        if (valid) {
                            uint32_t pk[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                pk[j] = pack_bf16x2(silu_mul(__uint_as_float(gv[2 * j]), __uint_as_float(uv[2 * j])),
                                                    silu_mul(__uint_as_float(gv[2 * j + 1]), __uint_as_float(uv[2 * j + 1])));
                            uint4* d4 = reinterpret_cast<uint4*>(out + grow * g.ldo + tl.n0 + c);
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                d4[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                        }
                    }
                } else {
                    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out);
                    for (int c = 0; c < g.bn; c += 32) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(tb + c, v);
                        tmem_ld_wait();
                        if (valid) {
                            uint32_t pk[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
                            uint4* d4 = reinterpret_cast<uint4*>(out + grow * g.ldo + tl.n0 + c);
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                d4[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                        }
                    }
                }
            } else {
                // weight tile: one TMEM lane = one output feature, one column = one row of the
                // expert's group
                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out);
                const int i = q * 32 + lane;  // weight row within the tile
                if (MODE == MODE_SWIGLU) {
                    // lane i: gate of feature n0 + i in columns [0, 128), its up in [128, 256)
                    const int feat = tl.n0 + i;
                    const bool fvalid = feat < g.n_out;
                    for (int c0 = 0; c0 < tl.ntok; c0 += 32) {
                        uint32_t gv[32], uv[32];
                        tmem_ld_32x32b_x32(tb + c0, gv);
                        tmem_ld_32x32b_x32(tb + 128 + c0, uv);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int row = c0 + j;
                            const int64_t grow = tl.row0 + row;
                            if (fvalid && row < tl.rows && grow < g.rows_cap)
                                out[grow * g.ldo + feat] = __float2bfloat16_rn(
                                    silu_mul(__uint_as_float(gv[j]), __uint_as_float(uv[j])));
                        }
                    }
                } else {
                    const int feat = tl.n0 + i;
                    const bool fvalid = feat < g.n_out;
                    for (int c0 = 0; c0 < tl.ntok; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(tb + c0, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int row = c0 + j;
                            const int64_t grow = tl.row0 + row;
                            if (fvalid && row < tl.rows && grow < g.rows_cap)
                                out[grow * g.ldo + feat] = __float2bfloat16_rn(__uint_as_float(v[j]));
                        }
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

// ------------------------------------------------------------------------------ host side --

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

// Row-major bf16 matrix [rows, cols] read in boxes of box_rows x 64 with the 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
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

template <int MODE>
cudaError_t launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& msa,
                        const CUtensorMap& msb, const GemmArgs& args, int grid, cudaStream_t st) {
    const size_t smem = SmemLayout::bytes(args.n_groups);
    static int configured_bytes[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && configured_bytes[dev] < static_cast<int>(smem)) {
        // always raise to the kernel's maximum once, so later calls skip this
        int max_optin = 0;
        e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return e;
        if (static_cast<int>(smem) > max_optin) return cudaErrorInvalidValue;
        e = cudaFuncSetAttribute(umma_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 max_optin);
        if (e != cudaSuccess) return e;
        configured_bytes[dev] = max_optin;
    }
    umma_gemm_kernel<MODE><<<grid, NUM_THREADS, smem, st>>>(ma, mb, msa, msb, args);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_gemm(const void* x, const void* wr, float* logits, int T, int d, int E,
                               uint32_t* status, cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    int bn = ((E + 31) / 32) * 32;
    if (bn > 256) bn = 256;
    CUtensorMap ma, mb;
    if (!make_map(&ma, x, static_cast<uint64_t>(T), d, BM)) return cudaErrorInvalidValue;
    if (!make_map(&mb, wr, static_cast<uint64_t>(E), d, bn)) return cudaErrorInvalidValue;
    GemmArgs a{};
    a.offsets = nullptr;
    a.out = logits;
    a.status = status;
    a.wait_ns = wait_limit_ns();
    a.rows_cap = T;
    a.ldo = E;
    a.n_groups = 1;
    a.rows = T;
    a.kdim = d;
    a.n_out = E;
    a.bn = bn;
    a.tile_cols = bn;
    a.ntiles = (E + bn - 1) / bn;
    a.s_cols = 0;
    const int tiles = ((T + BM - 1) / BM) * a.ntiles;
    const int grid = tiles < di->sm_count ? tiles : di->sm_count;
    return launch_gemm<MODE_ROUTER>(ma, mb, ma, mb, a, grid, st);
}

cudaError_t launch_grouped_swiglu(const void* x_perm, int64_t rows_cap, const int32_t* offsets,
                                  int N, const void* w13, int d, int I, void* h, uint32_t* status,
                                  cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    const int half = (I % 128 == 0) ? 128 : 64;
    CUtensorMap ma, mb, msa, msb;
    if (!make_map(&ma, x_perm, static_cast<uint64_t>(rows_cap), d, BM)) return cudaErrorInvalidValue;
    if (!make_map(&mb, w13, static_cast<uint64_t>(N) * 2 * I, d, half)) return cudaErrorInvalidValue;
    if (!make_map(&msa, w13, static_cast<uint64_t>(N) * 2 * I, d, 128)) return cudaErrorInvalidValue;
    if (!make_map(&msb, x_perm, static_cast<uint64_t>(rows_cap), d, SWAP_BOX)) return cudaErrorInvalidValue;
    GemmArgs a{};
    a.offsets = offsets;
    a.out = h;
    a.status = status;
    a.wait_ns = wait_limit_ns();
    a.rows_cap = rows_cap;
    a.ldo = I;
    a.n_groups = N;
    a.rows = 0;
    a.kdim = d;
    a.n_out = I;
    a.bn = 2 * half;
    a.tile_cols = half;
    a.ntiles = I / half;
    a.b_group_rows = 2 * I;
    a.up_off = I;
    a.s_cols = 128;  // 128 features (128 gate + 128 up rows); the last tile may pass I: masked
    a.s_tiles = (I + 127) / 128;
    return launch_gemm<MODE_SWIGLU>(ma, mb, msa, msb, a, di->sm_count, st);
}

cudaError_t launch_grouped_down(const void* h, int64_t rows_cap, const int32_t* offsets, int N,
                                const void* w2, int d, int I, void* y, uint32_t* status,
                                cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    const int bn = (d % 256 == 0) ? 256 : (d % 128 == 0) ? 128 : 64;
    CUtensorMap ma, mb, msa, msb;
    if (!make_map(&ma, h, static_cast<uint64_t>(rows_cap), I, BM)) return cudaErrorInvalidValue;
    if (!make_map(&mb, w2, static_cast<uint64_t>(N) * d, I, bn)) return cudaErrorInvalidValue;
    if (!make_map(&msa, w2, static_cast<uint64_t>(N) * d, I, 128)) return cudaErrorInvalidValue;
    if (!make_map(&msb, h, static_cast<uint64_t>(rows_cap), I, SWAP_BOX)) return cudaErrorInvalidValue;
    GemmArgs a{};
    a.offsets = offsets;
    a.out = y;
    a.status = status;
    a.wait_ns = wait_limit_ns();
    a.rows_cap = rows_cap;
    a.ldo = d;
    a.n_groups = N;
    a.rows = 0;
    a.kdim = I;
    a.n_out = d;
    a.bn = bn;
    a.tile_cols = bn;
    a.ntiles = d / bn;
    a.b_group_rows = d;
    a.up_off = 0;
    a.s_cols = 128;  // 128 output features per weight tile (the last may pass d: masked)
    a.s_tiles = (d + 127) / 128;
    return launch_gemm<MODE_DOWN>(ma, mb, msa, msb, a, di->sm_count, st);
}

}  // namespace lcmoe
