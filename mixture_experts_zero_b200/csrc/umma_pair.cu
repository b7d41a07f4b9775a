// umma_pair.cu -- the grouped expert GEMMs on CTA pairs (tcgen05.mma.cta_group::2).
//
//   grouped GEMM 1: H[rows_e, I] (bf16) = silu(X_e Wg[e]^T) * (X_e Wu[e]^T)   (SwiGLU epilogue)
//   grouped GEMM 2: Y[rows_e, d] (bf16) = H_e Wd[e]^T
// for the N FFN experts of the MoE equation (LongCat-Flash llm-wiki entity page, section 2.1);
// rows routed to zero-computation experts never reach these GEMMs.
//
// A cluster of two CTAs (one per SM) computes 256-row MMA tiles: each CTA holds 128 rows of the
// A operand and half of the B operand in its own shared memory, and the pair leader issues
// 256 x N x 16 MMAs that read both; each CTA's TMEM receives its 128 rows of the accumulator.
// Per SM this halves the B bytes loaded per FLOP compared with a 128-row tile, which lowers the
// L2-to-SM traffic of the main loop by a third.
//
// Roles (384 threads per CTA):
//   warp 0, one lane, both CTAs  TMA producer: loads this CTA's share of each stage; the bytes
//                                 complete on the leader's full barrier, where the leader alone
//                                 posts the expected byte count of the pair;
//   warp 1, one lane, leader     MMA issuer; tcgen05.commit with a 2-CTA multicast releases the
//                                 stage in both CTAs and publishes finished accumulators to both;
//   warp 1, both CTAs            TMEM allocation / deallocation (512 columns, cta_group::2);
//   warps 4..11, both CTAs       two epilogue groups of four warps; group g drains accumulator g
//                                 (TMEM columns [256 g, 256 g + 256)) over this CTA's 128 lanes,
//                                 and each of its warps arrives on the leader's accumulator-empty
//                                 barrier g (8 arrivals: 4 warps in each CTA).
//
// Tile kinds:
//   row tiles: 256 rows of one expert. GEMM 1: the leader loads 128 gate rows and its peer the
//     matching 128 up rows of B, so accumulator columns [0, 128) hold gate and [128, 256) hold up
//     values for every row. GEMM 2: 256 output features, 128 per CTA. A "wide" row tile (when I is
//     a multiple of 256 for GEMM 1, d a multiple of 512 for GEMM 2) loads a second box of B rows
//     one tile width further on and issues a second MMA on the same A into the other accumulator:
//     256 rows x 512 accumulator columns per tile, so the row operand is read once per 512
//     columns instead of once per 256, a quarter fewer bytes from L2 per FLOP. Its two halves
//     are drained by the two epilogue groups in parallel.
//   weight tiles ("swap"): 256 weight rows (128 per CTA) on the M side and the rows of one expert,
//     rounded up to 16 and split between the CTAs, on the N side (N <= 128; the kernel handles
//     N up to 256 in GEMM 2 should rem_rows be raised). GEMM 1 issues a gate MMA into columns
//     [0, N) and an up MMA into [128, 128 + N).
//     A GEMM 2 weight tile of N <= 128 is "double" (when d is a multiple of 512): it loads two
//     boxes of weight rows per k-step, 256 output features apart, and issues their MMAs on the
//     same token rows into columns [0, N) and [128, 128 + N): 512 features per tile, so a stage
//     carries twice the weight bytes per token byte and the ring keeps twice the weight bytes in
//     flight of a plain weight tile (the cold experts' tiles are a weight stream whose rate per
//     SM is set by the bytes in flight).
// Accumulators: a wide row tile takes both; every other tile takes the next one in turn, so the
// epilogue of one weight tile or narrow row tile overlaps the main loop of the next.
// Per expert with c_e rows: below cold_rows it is "cold" and runs as weight tiles only; otherwise
// it runs floor(c_e / 256) row tiles, and its leftover rows run as one more row tile if there are
// at least rem_rows of them, else as weight tiles (N rounded up to 16). Both GEMMs: cold_rows =
// rem_rows = 128, so every weight tile has N <= 128 (a GEMM 2 weight tile is then double when d
// is a multiple of 512). The tile list (built on the device from offsets, identically by every
// CTA) is: for each hot expert in order, its row tiles (every row block of its first slice of
// output features, then of the next slice, ...) then its leftover weight tiles; then the weight
// tiles of every cold expert.
// Tiles are handed out in list order as pairs become free: as the leader's producer starts a
// tile it takes the index of its next one from a counter in global memory (zeroed before each
// launch), and it passes each index to every role of both CTAs through a queue of TQ tile
// indices in shared memory
// (a full barrier per slot in each CTA, released by the leader's producer; an empty barrier per
// slot in the leader, which counts the 18 other readers: the MMA issuer, the eight epilogue warps
// of each CTA and the peer's producer). The tiles that share a hot expert's weights then start
// within microseconds of one another, so those weights are read from L2 rather than fetched again,
// and the pairs finish together. The index past the last tile ends every role's loop.
// Every wait is bounded (lc_moe_set_wait_limit_ns); a wait that runs out raises a CTA-wide abort,
// records LC_MOE_DEV_WAIT_TIMEOUT, drains in-flight copies and MMAs, and frees TMEM.
#include <cudaTypedefs.h>

#include <cstdlib>
#include <mutex>

#include "common.cuh"

namespace lcmoe {

namespace {

constexpr int HALF_M = 128;                 // A rows per CTA
constexpr int BK = 64;                      // 64 bf16 = 128 bytes = one swizzle row
constexpr int A_BYTES = HALF_M * BK * 2;    // 16 KB: one 128-row operand box of a k-step
constexpr int TMEM_COLS = 512;
constexpr int NUM_THREADS = 384;
constexpr int EPI_WARP0 = 4;              // warps 4..11: two epilogue groups of four warps
constexpr int TOK_BOX = 8;                  // token rows per TMA box of a weight tile (per CTA)
constexpr int TOK_ROUND = 2 * TOK_BOX;      // weight-tile N is a multiple of this
constexpr int TQ = 8;                       // depth of the tile-index queue

enum Mode : int { MODE_SWIGLU = 1, MODE_DOWN = 2 };

// Shared-memory ring, the same for both GEMMs: a stage holds the row box and two weight boxes (a
// wide row tile's two accumulators), a GEMM 1 weight tile's gate and up rows plus up to 64 token
// rows, a GEMM 2 double weight tile's two weight boxes plus up to 64 token rows, or a plain
// weight tile's box plus up to 128 token rows: 48 KB in 4 stages. `stages` is the depth when the
// per-expert tables fit beside it; for GEMM 2 launch_pair takes one stage fewer at a time until
// they do (very many experts).
template <int MODE>
struct Ring {
    static constexpr int stages = 4;
    static constexpr int bytes = 3 * A_BYTES;
};

struct PairArgs {
    const int32_t* offsets;  // [n_groups + 1] row offsets
    __nv_bfloat16* out;      // [rows_cap, ldo]
    uint32_t* status;
    uint64_t wait_ns;
    int64_t rows_cap;
    int64_t ldo;
    int n_groups;
    int kdim;                // reduction length (multiple of 64)
    int n_out;               // output columns (I or d)
    int ntiles;              // row tiles per 256-row block of an expert
    int tile_cols;           // output columns per row tile
    int b_group_rows;        // rows of the weight matrix per expert
    int up_off;              // GEMM 1: row offset of Wu inside an expert (= I)
    int s_tiles;             // weight tiles per group of rows (256 output features each)
    int cold_rows;           // experts with 0 < rows < cold_rows use weight tiles only
    int rem_rows;            // an expert's rows past its last full 256-row tile: fewer than this
                             // run as weight tiles, otherwise as one more row tile
    int wide;                // row tiles span two accumulators (2 * tile_cols output columns)
    int dbl;                 // GEMM 2: weight tiles of N <= 128 cover 512 output features
    int stages;              // ring depth (set by launch_pair)
    const float* row_scale;  // E4M3 GEMM 1: scale of each grouped row [rows_cap]
    const float* w_scale;    // E4M3 GEMM 1: scale of each weight row [n_groups * b_group_rows]
    int64_t abort_kstep;     // test switch: the MMA issuer gives up before this k-step (< 0: never)
    unsigned long long* clock_probe;  // [4] start ns, start cycles, end ns, end cycles of CTA 0
    int* tile_ctr;           // next tile index (zeroed before each launch; in the status area)
};

// Epilogue transpose tile of one warp: 32 rows x 32 features (bf16), 64 bytes per row, its four
// 16-byte chunks stored at chunk ^ ((row >> 1) & 3), so that both the writes (one row at a time)
// and the reads (8 rows per 128-byte phase) hit distinct banks.
constexpr int XPOSE_ROW = 64;
constexpr int XPOSE_WARP = 32 * XPOSE_ROW;

// Shared memory of one CTA with a ring of `st` stages: the ring, the barriers (full and empty per
// stage, tfull[2], tempty[2], drain), the TMEM address and abort flag, the tile-index queue (full
// and empty barriers, TQ indices), the epilogue transpose tiles, the per-expert tile prefix sums.
template <int MODE>
struct Layout {
    int bars_off, misc_off, xpose_off, table_off;
    __host__ __device__ explicit Layout(int st)
        : bars_off(st * Ring<MODE>::bytes),
          misc_off(bars_off + (2 * st + 5) * 8),
          xpose_off((misc_off + 16 + 2 * TQ * 8 + TQ * 4 + 127) & ~127),
          table_off(xpose_off + 8 * XPOSE_WARP) {}
    size_t bytes(int n_groups) const { return 1024 + table_off + 2 * static_cast<size_t>(n_groups + 1) * 4; }
};

struct Tile {
    int swap;
    int wide;  // row tile over both accumulators
    int dbl;   // double weight tile (GEMM 2, 512 output features)
    int grp;
    int64_t row0;
    int rows;
    int n0;
    int ntok;  // weight tile: MMA N
};

// Which TMEM accumulators (two of 256 columns) each tile uses, followed identically by the MMA
// issuer and the two epilogue groups: a wide row tile takes both; every other tile takes the
// next one in turn. Bit b of `phase` is the parity of buffer b's current use.
struct AccSchedule {
    int next = 0;
    uint32_t phase = 0u;
    __device__ __forceinline__ int buffers(int wide) const { return wide ? 3 : (1 << next); }
    __device__ __forceinline__ uint32_t parity(int b) const { return (phase >> b) & 1u; }
    __device__ __forceinline__ void advance(int wide) {
        phase ^= static_cast<uint32_t>(buffers(wide));
        if (!wide) next ^= 1;
    }
};

__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// silu(g) * u. The quotient is the fast division (within 2 ulp of fp32, and 0 once 1 + e^-g
// passes 2^126, where silu(g) is below 2^-119): the IEEE division routine made the SwiGLU
// epilogue three times longer (15 against 5 us per 128 x 128 block), and H is rounded to bf16.
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// Row tile store of one warp's 32-row x 32-feature bf16 block, held one row per lane (pk: the
// lane's 64 bytes). The block goes through the warp's transpose buffer, so that each store
// instruction writes eight whole 64-byte row segments instead of 32 scattered 16-byte pieces.
// Rows nv .. 31 are skipped; dst = the block's first output element (row of lane 0); the whole
// warp calls it.
__device__ __forceinline__ void store_row_block(uint8_t* xp, const uint32_t (&pk)[16], int nv,
                                                __nv_bfloat16* dst, int64_t ldo) {
    const int lane = threadIdx.x & 31;
    if (lane < nv) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(xp + lane * XPOSE_ROW + (((j ^ (lane >> 1)) & 3) << 4)) =
                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
    }
    __syncwarp();
    const int k = lane & 3;
#pragma unroll
    for (int i2 = 0; i2 < 4; ++i2) {
        const int rr = (lane >> 2) + 8 * i2;
        if (rr < nv)
            *reinterpret_cast<uint4*>(dst + rr * ldo + k * 8) =
                *reinterpret_cast<const uint4*>(xp + rr * XPOSE_ROW + (((k ^ (rr >> 1)) & 3) << 4));
    }
    __syncwarp();
}

template <bool F8>
__device__ __forceinline__ void mma_step(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    if (F8) umma_e4m3_pair(d_tmem, adesc, bdesc, idesc, accumulate);
    else umma_bf16_pair(d_tmem, adesc, bdesc, idesc, accumulate);
}

__device__ __forceinline__ int upper_group(const int32_t* pre, int n, int v) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= v) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// F8: operands are E4M3 codes (GEMM 1 only): a 128-byte k-step holds 128 elements, the MMAs are
// kind::f8f6f4 (K = 32 per instruction), and the epilogue multiplies each accumulator by its row's
// scale and its weight row's scale before the SwiGLU.
template <int MODE, bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    umma_pair_kernel(const __grid_constant__ CUtensorMap mapRows, const __grid_constant__ CUtensorMap mapW,
                     const __grid_constant__ CUtensorMap mapTok, const PairArgs g) {
    // GEMM 1's depth is fixed (its tables always fit); GEMM 2's is set per launch
    const int STAGES = MODE == MODE_DOWN ? g.stages : Ring<MODE>::stages;
    constexpr int STAGE_BYTES = Ring<MODE>::bytes;
    const Layout<MODE> L(STAGES);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars_off);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc_off);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc_off + 4);
    // tile-index queue (see the header comment)
    uint64_t* tq_full = reinterpret_cast<uint64_t*>(smem + L.misc_off + 16);
    uint64_t* tq_empty = tq_full + TQ;
    int* tq = reinterpret_cast<int*>(tq_empty + TQ);
    // group row offsets are read from global memory (L1-resident after the first tiles); shared
    // memory holds the per-expert tile prefix sums
    const int32_t* __restrict__ offs = g.offsets;
    int32_t* rpre_s = reinterpret_cast<int32_t*>(smem + L.table_off);
    int32_t* spre_s = rpre_s + (g.n_groups + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 8);  // 4 epilogue warps in each CTA of the pair
        }
        mbar_init(drain, 1);
        for (int i = 0; i < TQ; ++i) {
            mbar_init(&tq_full[i], 1);
            mbar_init(&tq_empty[i], 18);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&mapRows);
        tma_prefetch_desc(&mapW);
        tma_prefetch_desc(&mapTok);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    __syncthreads();
    if (warp == 2) {
        // per expert: tiles of the hot part (row tiles + weight tiles of the leftover rows) and
        // weight tiles of a cold expert; exclusive prefix sums of both
        int run_h = 0, run_c = 0;
        if (lane == 0) {
            rpre_s[0] = 0;
            spre_s[0] = 0;
        }
        for (int base = 0; base < g.n_groups; base += 32) {
            const int e = base + lane;
            int nh = 0, nc = 0;
            if (e < g.n_groups) {
                int cnt = __ldg(offs + (e + 1)) - __ldg(offs + (e));
                if (cnt < 0) {
                    cnt = 0;
                    set_status(g.status, LC_MOE_DEV_IDX_RANGE);
                }
                if (cnt > 0 && cnt < g.cold_rows) {
                    nc = (g.dbl && cnt <= HALF_M) ? g.s_tiles / 2 : g.s_tiles;
                } else if (cnt > 0) {
                    const int nfull = cnt / (2 * HALF_M);
                    const int rem = cnt - nfull * 2 * HALF_M;
                    const bool rem_row = rem >= g.rem_rows;
                    nh = (nfull + (rem_row ? 1 : 0)) * g.ntiles;
                    if (rem > 0 && !rem_row) nh += (g.dbl && rem <= HALF_M) ? g.s_tiles / 2 : g.s_tiles;
                }
            }
            int ih = nh, ic = nc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int vh = __shfl_up_sync(0xffffffffu, ih, o);
                const int vc = __shfl_up_sync(0xffffffffu, ic, o);
                if (lane >= o) {
                    ih += vh;
                    ic += vc;
                }
            }
            if (e < g.n_groups) {
                rpre_s[e + 1] = run_h + ih;
                spre_s[e + 1] = run_c + ic;
            }
            run_h += __shfl_sync(0xffffffffu, ih, 31);
            run_c += __shfl_sync(0xffffffffu, ic, 31);
        }
    }
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers are initialised before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    if (g.clock_probe && blockIdx.x == 0 && threadIdx.x == 0) {
        g.clock_probe[0] = globaltimer_ns();
        g.clock_probe[1] = clock64();
    }

    const int total_r = rpre_s[g.n_groups];
    const int total_s = spre_s[g.n_groups];
    const int total = total_r + total_s;
    constexpr int KB = F8 ? 2 * BK : BK;  // elements per 128-byte k-step
    const int nk = g.kdim / KB;

    auto decode = [&](int tile) {
        Tile tl;
        if (tile < total_r) {
            // hot expert: its row tiles, then weight tiles for the rows past its last row tile
            const int e = upper_group(rpre_s, g.n_groups, tile);
            const int local = tile - rpre_s[e];
            const int cnt = __ldg(offs + (e + 1)) - __ldg(offs + (e));
            const int nfull = cnt / (2 * HALF_M);
            const int rem = cnt - nfull * 2 * HALF_M;
            const int nrow = (nfull + (rem >= g.rem_rows ? 1 : 0)) * g.ntiles;
            tl.grp = e;
            tl.dbl = 0;
            if (local < nrow) {
                // feature-major: every row block of one slice of output features, then the next
                // slice, so the tiles that read the same weight slice are handed out together
                const int nblk = nrow / g.ntiles;
                const int mt = local % nblk;
                const int nt = local / nblk;
                tl.swap = 0;
                tl.wide = g.wide;
                tl.row0 = static_cast<int64_t>(__ldg(offs + (e))) + static_cast<int64_t>(mt) * 2 * HALF_M;
                tl.rows = min(2 * HALF_M, cnt - mt * 2 * HALF_M);
                tl.n0 = nt * g.tile_cols * (g.wide ? 2 : 1);
                tl.ntok = 0;
            } else {
                tl.swap = 1;
                tl.wide = 0;
                tl.row0 = static_cast<int64_t>(__ldg(offs + (e))) + static_cast<int64_t>(nfull) * 2 * HALF_M;
                tl.rows = rem;
                tl.dbl = g.dbl && rem <= HALF_M;
                tl.n0 = (local - nrow) * (tl.dbl ? 4 : 2) * HALF_M;
                tl.ntok = (rem + TOK_ROUND - 1) / TOK_ROUND * TOK_ROUND;
            }
        } else {
            // cold expert: weight tiles only
            const int idx = tile - total_r;
            const int e = upper_group(spre_s, g.n_groups, idx);
            tl.swap = 1;
            tl.wide = 0;
            tl.grp = e;
            tl.row0 = __ldg(offs + (e));
            tl.rows = __ldg(offs + (e + 1)) - __ldg(offs + (e));
            tl.dbl = g.dbl && tl.rows <= HALF_M;
            tl.n0 = (idx - spre_s[e]) * (tl.dbl ? 4 : 2) * HALF_M;
            tl.ntok = (tl.rows + TOK_ROUND - 1) / TOK_ROUND * TOK_ROUND;
        }
        return tl;
    };

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------- TMA producer (both CTAs) --
        const uint64_t pol_stream = l2_policy_evict_first();
        const uint64_t pol_normal = l2_policy_evict_normal();
        int s = 0;
        uint32_t ph = 0;
        int issued = 0;
        bool ok = true;
        int nxt = leader ? atomicAdd(g.tile_ctr, 1) : 0;
        for (int qi = 0; ok; ++qi) {
            const int slot = qi % TQ;
            const uint32_t par = (qi / TQ) & 1;
            int tile;
            if (leader) {
                if (qi >= TQ && !mbar_wait_cluster(&tq_empty[slot], par ^ 1u, g.wait_ns, abort_flag, g.status)) {
                    ok = false;
                    break;
                }
                tile = nxt < total ? nxt : total;
                tq[slot] = tile;
                st_shared_cluster_u32(mapa_shared(smem_u32(&tq[slot]), 1), static_cast<uint32_t>(tile));
                mbar_arrive(&tq_full[slot]);
                mbar_arrive_cluster(mapa_shared(smem_u32(&tq_full[slot]), 1));
                if (tile < total) nxt = atomicAdd(g.tile_ctr, 1);
            } else {
                if (!mbar_wait_cluster(&tq_full[slot], par, g.wait_ns, abort_flag, g.status)) {
                    ok = false;
                    break;
                }
                tile = tq[slot];
                mbar_arrive_cluster(mapa_shared(smem_u32(&tq_empty[slot]), 0));
            }
            if (tile >= total) break;
            const Tile tl = decode(tile);
            const int tok_rows = tl.ntok / 2;  // this CTA's share of the N side
            uint32_t cta_bytes;
            if (!tl.swap) cta_bytes = (tl.wide ? 3 : 2) * A_BYTES;
            else cta_bytes = ((MODE == MODE_SWIGLU || tl.dbl) ? 2 : 1) * A_BYTES + tok_rows * BK * 2;
            const int wbase = tl.grp * g.b_group_rows;
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait(&empty[s], ph ^ 1u, g.wait_ns, abort_flag, g.status)) {
                    ok = false;
                    break;
                }
                uint8_t* sa = smem + s * STAGE_BYTES;
                uint8_t* sb = sa + A_BYTES;
                const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
                if (leader) mbar_arrive_expect_tx(&full[s], 2 * cta_bytes);
                const int kx = kb * KB;
                if (!tl.swap) {
                    tma_load_2d_pair(sa, &mapRows, bar, kx, static_cast<int32_t>(tl.row0 + rank * HALF_M), pol_normal);
                    // GEMM 1: leader gate rows, peer up rows; GEMM 2: 128 output features each
                    const int wrow = (MODE == MODE_SWIGLU) ? wbase + tl.n0 + static_cast<int>(rank) * g.up_off
                                                           : wbase + tl.n0 + static_cast<int>(rank) * HALF_M;
                    tma_load_2d_pair(sb, &mapW, bar, kx, wrow, pol_normal);
                    // wide tile: the weight rows of the second accumulator (the next tile_cols
                    // output columns), one box further on
                    if (tl.wide) tma_load_2d_pair(sb + A_BYTES, &mapW, bar, kx, wrow + g.tile_cols, pol_normal);
                } else {
                    const int wrow = wbase + tl.n0 + static_cast<int>(rank) * HALF_M;
                    tma_load_2d_pair(sa, &mapW, bar, kx, wrow, pol_stream);
                    uint8_t* st = sb;
                    if (MODE == MODE_SWIGLU || tl.dbl) {
                        // GEMM 1: the up rows of the same features; double tile: the weight rows
                        // 256 features further on
                        tma_load_2d_pair(sb, &mapW, bar, kx, wrow + (MODE == MODE_SWIGLU ? g.up_off : 2 * HALF_M),
                                         pol_stream);
                        st = sb + A_BYTES;
                    }
                    const int64_t t0 = tl.row0 + static_cast<int64_t>(rank) * tok_rows;
                    for (int b = 0; b < tok_rows; b += TOK_BOX)
                        tma_load_2d_pair(st + b * 128, &mapTok, bar, kx, static_cast<int32_t>(t0 + b), pol_normal);
                }
                ++issued;
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        if (!ok && leader) {
            for (int i = 0; i < STAGES && i < issued; ++i) {
                if (s == 0) {
                    s = STAGES - 1;
                    ph ^= 1u;
                } else {
                    --s;
                }
                wait_drain(&full[s], ph, g.wait_ns);
            }
        }
    } else if (warp == 1 && lane == 0 && leader) {
        // ------------------------------------------------------- MMA issuer (leader only) --
        int s = 0;
        uint32_t ph = 0;
        AccSchedule sched;
        bool ok = true;
        int64_t ksteps = 0;
        for (int qi = 0; ok; ++qi) {
            const int slot = qi % TQ;
            if (!mbar_wait(&tq_full[slot], (qi / TQ) & 1, g.wait_ns, abort_flag, g.status)) break;
            const int tile = tq[slot];
            mbar_arrive(&tq_empty[slot]);
            if (tile >= total) break;
            const Tile tl = decode(tile);
            const uint32_t idesc = F8 ? idesc_e4m3_f32(2 * HALF_M, tl.swap ? tl.ntok : 2 * HALF_M)
                                      : idesc_bf16_f32(2 * HALF_M, tl.swap ? tl.ntok : 2 * HALF_M);
            const int bufs = sched.buffers(tl.wide);
            for (int b = 0; b < 2 && ok; ++b)
                if ((bufs >> b) & 1) ok = mbar_wait(&tempty[b], sched.parity(b) ^ 1u, g.wait_ns, abort_flag, g.status);
            if (!ok) break;
            tc_fence_after();
            const int acc = tl.wide ? 0 : sched.next;
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
            for (int kb = 0; kb < nk; ++kb) {
                if (ksteps++ == g.abort_kstep) {
                    // as if this stage's wait had run out: the abort and drain paths of every role
                    *abort_flag = 1;
                    set_status(g.status, LC_MOE_DEV_WAIT_TIMEOUT);
                    ok = false;
                    break;
                }
                if (!mbar_wait(&full[s], ph, g.wait_ns, abort_flag, g.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t* sa = smem + s * STAGE_BYTES;
                const uint64_t ad = sw128_kmajor_desc(smem_u32(sa));
                const uint64_t bd = sw128_kmajor_desc(smem_u32(sa + A_BYTES));
                if (tl.swap && (MODE == MODE_SWIGLU || tl.dbl)) {
                    const uint64_t td = sw128_kmajor_desc(smem_u32(sa + 2 * A_BYTES));
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        mma_step<F8>(d_tmem, ad + 2 * kk, td + 2 * kk, idesc, (kb | kk) != 0);
                        mma_step<F8>(d_tmem + 128, bd + 2 * kk, td + 2 * kk, idesc, (kb | kk) != 0);
                    }
                } else if (tl.wide) {
                    // second accumulator: the weight rows one box further on in shared memory
                    const uint64_t bd2 = sw128_kmajor_desc(smem_u32(sa + 2 * A_BYTES));
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        mma_step<F8>(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
                        mma_step<F8>(d_tmem + 256, ad + 2 * kk, bd2 + 2 * kk, idesc, (kb | kk) != 0);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_step<F8>(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
                }
                umma_commit_pair(&empty[s], 0x3);
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (!ok) break;
            for (int b = 0; b < 2; ++b)
                if ((bufs >> b) & 1) umma_commit_pair(&tfull[b], 0x3);
            sched.advance(tl.wide);
        }
        umma_commit_pair(drain, 0x1);
        wait_drain(drain, 0, g.wait_ns);
    } else if (warp >= EPI_WARP0) {
        // ------------------------------------------------------------ epilogue (both CTAs) --
        // group eg drains accumulator eg: its own tiles, or its half of a wide row tile; warp
        // w may only read TMEM lanes 32 * (w % 4) .. + 31
        const int q = warp & 3;
        const int eg = (warp - EPI_WARP0) >> 2;
        const int acc = eg;
        AccSchedule sched;
        __nv_bfloat16* out = g.out;
        for (int qi = 0;; ++qi) {
            const int slot = qi % TQ;
            if (!mbar_wait_cluster(&tq_full[slot], (qi / TQ) & 1, g.wait_ns, abort_flag, g.status)) break;
            const int tile = tq[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tq_empty[slot]), 0));
            if (tile >= total) break;
            const Tile tl = decode(tile);
            if (!((sched.buffers(tl.wide) >> acc) & 1)) {
                sched.advance(tl.wide);
                continue;
            }
            if (!mbar_wait(&tfull[acc], sched.parity(acc), g.wait_ns, abort_flag, g.status)) break;
            tc_fence_after();
            const uint32_t tb =
                tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * 256);
            const int i = q * 32 + lane;  // TMEM lane of this thread
            // first output column of this accumulator (the second half of a wide row tile starts
            // tile_cols further on)
            const int fbase = tl.n0 + (tl.wide ? acc * g.tile_cols : 0);
            if (!tl.swap) {
                const int r = static_cast<int>(rank) * HALF_M + i;  // row within the 256-row tile
                const int64_t grow = tl.row0 + r;
                const bool valid = r < tl.rows && grow < g.rows_cap;
                // the warp's 32 rows start at rb; nv of them are real rows
                const int rb = static_cast<int>(rank) * HALF_M + q * 32;
                int64_t nv64 = g.rows_cap - (tl.row0 + rb);
                if (nv64 > tl.rows - rb) nv64 = tl.rows - rb;
                const int nv = nv64 < 0 ? 0 : (nv64 > 32 ? 32 : static_cast<int>(nv64));
                uint8_t* xp = smem + L.xpose_off + (warp - EPI_WARP0) * XPOSE_WARP;
                __nv_bfloat16* out_rb = out + (tl.row0 + rb) * g.ldo;
                if (MODE == MODE_SWIGLU) {
                    // the next 32 columns' TMEM loads are in flight while this block is computed
                    uint32_t gbuf[2][32], ubuf[2][32];
                    tmem_ld_32x32b_x32(tb, gbuf[0]);
                    tmem_ld_32x32b_x32(tb + HALF_M, ubuf[0]);
#pragma unroll
                    for (int ci = 0; ci < HALF_M / 32; ++ci) {
                        const int c = ci * 32;
                        tmem_ld_wait();
                        if (ci + 1 < HALF_M / 32) {
                            tmem_ld_32x32b_x32(tb + c + 32, gbuf[(ci + 1) & 1]);
                            tmem_ld_32x32b_x32(tb + HALF_M + c + 32, ubuf[(ci + 1) & 1]);
                        }
                        uint32_t (&gv)[32] = gbuf[ci & 1];
                        uint32_t (&uv)[32] = ubuf[ci & 1];
                        const int f0 = fbase + c;
                        uint32_t pk[16];
                        if (valid && f0 < g.n_out) {
                            if (F8) {
                                // (acc * row scale) * weight-row scale, gate and up separately
                                const float sr = __ldg(g.row_scale + grow);
                                const float4* sg4 = reinterpret_cast<const float4*>(
                                    g.w_scale + static_cast<int64_t>(tl.grp) * g.b_group_rows + f0);
                                const float4* su4 = reinterpret_cast<const float4*>(
                                    g.w_scale + static_cast<int64_t>(tl.grp) * g.b_group_rows + g.up_off + f0);
#pragma unroll
                                for (int j4 = 0; j4 < 8; ++j4) {
                                    const float4 a = __ldg(sg4 + j4), b = __ldg(su4 + j4);
                                    const float sa[4] = {a.x, a.y, a.z, a.w}, sb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                                    for (int u = 0; u < 4; ++u) {
                                        gv[4 * j4 + u] = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(gv[4 * j4 + u]), sr), sa[u]));
                                        uv[4 * j4 + u] = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(uv[4 * j4 + u]), sr), sb[u]));
                                    }
                                }
                            }
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                pk[j] = pack_bf16x2(silu_mul(__uint_as_float(gv[2 * j]), __uint_as_float(uv[2 * j])),
                                                    silu_mul(__uint_as_float(gv[2 * j + 1]), __uint_as_float(uv[2 * j + 1])));
                        }
                        if (nv > 0 && f0 < g.n_out) store_row_block(xp, pk, nv, out_rb + f0, g.ldo);
                    }
                } else {
                    for (int c = 0; c < 2 * HALF_M; c += 32) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(tb + c, v);
                        tmem_ld_wait();
                        const int f0 = fbase + c;
                        uint32_t pk[16];
                        if (valid && f0 < g.n_out) {
                            if (F8) {
                                // (acc * row scale) * weight-row scale
                                const float sr = __ldg(g.row_scale + grow);
                                const float4* sw4 = reinterpret_cast<const float4*>(
                                    g.w_scale + static_cast<int64_t>(tl.grp) * g.b_group_rows + f0);
#pragma unroll
                                for (int j4 = 0; j4 < 8; ++j4) {
                                    const float4 a = __ldg(sw4 + j4);
                                    const float sa[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                                    for (int u = 0; u < 4; ++u)
                                        v[4 * j4 + u] = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(v[4 * j4 + u]), sr), sa[u]));
                                }
                            }
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
                        }
                        if (nv > 0 && f0 < g.n_out) store_row_block(xp, pk, nv, out_rb + f0, g.ldo);
                    }
                }
            } else {
                // weight tile: lane = output feature, column = row of the expert's group. Each
                // 32 x 32 block goes through shared memory transposed, so that every thread then
                // stores 32 consecutive features of one row as four 16-byte vectors.
                // A double weight tile's second 256 features are in columns [128, 128 + N).
                uint8_t* xp = smem + L.xpose_off + (warp - EPI_WARP0) * XPOSE_WARP;
                for (int half = 0; half < ((MODE == MODE_DOWN && tl.dbl) ? 2 : 1); ++half) {
                const int f0 = tl.n0 + half * 2 * HALF_M + static_cast<int>(rank) * HALF_M + q * 32;  // warp's first feature
                const uint32_t tbh = tb + static_cast<uint32_t>(half * HALF_M);
                for (int c0 = 0; c0 < tl.ntok; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tbh + c0, v);
                    if (MODE == MODE_SWIGLU) {
                        uint32_t uv[32];
                        tmem_ld_32x32b_x32(tbh + HALF_M + c0, uv);
                        tmem_ld_wait();
                        if (F8) {
                            // lane = weight row (feature), column j = grouped row c0 + j
                            const int64_t wb = static_cast<int64_t>(tl.grp) * g.b_group_rows;
                            const int fl = f0 + lane < g.n_out ? f0 + lane : g.n_out - 1;
                            const float sg = __ldg(g.w_scale + wb + fl);
                            const float su = __ldg(g.w_scale + wb + g.up_off + fl);
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                int64_t rr = tl.row0 + c0 + j;
                                if (rr >= g.rows_cap) rr = g.rows_cap - 1;
                                const float sr = __ldg(g.row_scale + rr);
                                v[j] = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(v[j]), sr), sg));
                                uv[j] = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(uv[j]), sr), su));
                            }
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            v[j] = __float_as_uint(silu_mul(__uint_as_float(v[j]), __uint_as_float(uv[j])));
                    } else {
                        tmem_ld_wait();
                        if (F8) {
                            const int fl = f0 + lane < g.n_out ? f0 + lane : g.n_out - 1;
                            const float sw = __ldg(g.w_scale + static_cast<int64_t>(tl.grp) * g.b_group_rows + fl);
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                int64_t rr = tl.row0 + c0 + j;
                                if (rr >= g.rows_cap) rr = g.rows_cap - 1;
                                v[j] = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(v[j]), __ldg(g.row_scale + rr)), sw));
                            }
                        }
                    }
                    // lane = feature f0 + lane, v[j] = value for row c0 + j
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        *reinterpret_cast<__nv_bfloat16*>(
                            xp + j * XPOSE_ROW + ((((lane >> 3) ^ (j >> 1)) & 3) << 4) + (lane & 7) * 2) =
                            __float2bfloat16_rn(__uint_as_float(v[j]));
                    __syncwarp();
                    const int row = c0 + lane;
                    const int64_t grow = tl.row0 + row;
                    if (row < tl.rows && grow < g.rows_cap && f0 < g.n_out) {
                        uint4* dst = reinterpret_cast<uint4*>(out + grow * g.ldo + f0);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            dst[k] = *reinterpret_cast<const uint4*>(
                                xp + lane * XPOSE_ROW + (((k ^ (lane >> 1)) & 3) << 4));
                    }
                    __syncwarp();
                }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
            sched.advance(tl.wide);
        }
    }

    __syncthreads();
    cluster_sync_all();  // the leader's MMAs have finished reading the peer's shared memory
    if (g.clock_probe && blockIdx.x == 0 && threadIdx.x == 0) {
        g.clock_probe[2] = globaltimer_ns();
        g.clock_probe[3] = clock64();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

template <int MODE, bool F8>
cudaError_t launch_pair(const CUtensorMap& mr, const CUtensorMap& mw, const CUtensorMap& mt,
                        const PairArgs& args, int grid, cudaStream_t st) {
    if (MODE == MODE_SWIGLU && args.dbl) return cudaErrorInvalidValue;
    // once per device: allow the kernel the device's whole opt-in shared memory
    static PerDeviceOnce setup;
    static int max_optin[PerDeviceOnce::kMaxDevices];
    cudaError_t e = setup.run([](int dev) {
        int v = 0;
        cudaError_t r = cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (r != cudaSuccess) return r;
        r = cudaFuncSetAttribute(umma_pair_kernel<MODE, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, v);
        if (r == cudaSuccess) max_optin[dev] = v;
        return r;
    });
    if (e != cudaSuccess) return e;
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    // the ring as deep as the per-expert tables leave room for (at least two stages)
    PairArgs a = args;
    a.stages = Ring<MODE>::stages;
    if (MODE == MODE_DOWN)
        while (a.stages > 2 && Layout<MODE>(a.stages).bytes(a.n_groups) > static_cast<size_t>(max_optin[dev])) --a.stages;
    const size_t smem = Layout<MODE>(a.stages).bytes(a.n_groups);
    if (smem > static_cast<size_t>(max_optin[dev])) return cudaErrorInvalidValue;
    if ((e = cudaMemsetAsync(a.tile_ctr, 0, sizeof(int), st)) != cudaSuccess) return e;
    umma_pair_kernel<MODE, F8><<<grid, NUM_THREADS, smem, st>>>(mr, mw, mt, a);
    return cudaGetLastError();
}

int pair_grid(const DevInfo* di) { return (di->sm_count / 2) * 2; }

// The k-step before which the MMA issuer of every grouped-GEMM launch gives up as if a wait had
// run out, from the environment variable LC_MOE_DEBUG_GEMM_ABORT_KSTEP (unset in normal use: never).
// It exists for the device test of the abort path: the other roles then leave through the abort
// flag or their own bounded waits, drain what they issued and free TMEM.
int64_t debug_abort_kstep() {
    const char* v = std::getenv("LC_MOE_DEBUG_GEMM_ABORT_KSTEP");
    if (!v || !*v) return -1;
    char* end = nullptr;
    const long long k = std::strtoll(v, &end, 10);
    return (end && *end == '\0' && k >= 0) ? static_cast<int64_t>(k) : -1;
}

}  // namespace

namespace {

PairArgs swiglu_args(int64_t rows_cap, const int32_t* offsets, int N, int d, int I, void* h,
                     uint32_t* status) {
    PairArgs a{};
    a.offsets = offsets;
    a.out = static_cast<__nv_bfloat16*>(h);
    a.status = status;
    a.wait_ns = wait_limit_ns();
    a.clock_probe = clock_probe();
    a.tile_ctr = reinterpret_cast<int*>(status + 16);
    a.abort_kstep = debug_abort_kstep();
    a.rows_cap = rows_cap;
    a.ldo = I;
    a.n_groups = N;
    a.kdim = d;
    a.n_out = I;
    // 128 features (gate + up) per accumulator; when I allows, a row tile covers 256 features
    // in both accumulators (wide), which halves the row-operand reads per FLOP
    a.tile_cols = HALF_M;
    a.wide = (I % (2 * HALF_M) == 0) ? 1 : 0;
    a.ntiles = a.wide ? I / (2 * HALF_M) : (I + HALF_M - 1) / HALF_M;
    a.b_group_rows = 2 * I;
    a.up_off = I;
    a.s_tiles = (I + 2 * HALF_M - 1) / (2 * HALF_M);  // 256 features per weight tile
    // weight-tile N <= 128 keeps gate and up in one 256-column accumulator
    a.cold_rows = 128;
    a.rem_rows = 128;
    return a;
}

}  // namespace

cudaError_t launch_grouped_swiglu(const void* x_perm, int64_t rows_cap, const int32_t* offsets,
                                  int N, const void* w13, int d, int I, void* h, uint32_t* status,
                                  cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    CUtensorMap mr, mw, mt;
    if (!make_tma_map_2d(&mr, x_perm, static_cast<uint64_t>(rows_cap), d, HALF_M)) return cudaErrorInvalidValue;
    if (!make_tma_map_2d(&mw, w13, static_cast<uint64_t>(N) * 2 * I, d, HALF_M)) return cudaErrorInvalidValue;
    if (!make_tma_map_2d(&mt, x_perm, static_cast<uint64_t>(rows_cap), d, TOK_BOX)) return cudaErrorInvalidValue;
    const PairArgs a = swiglu_args(rows_cap, offsets, N, d, I, h, status);
    return launch_pair<MODE_SWIGLU, false>(mr, mw, mt, a, pair_grid(di), st);
}

cudaError_t launch_grouped_swiglu_e4m3(const void* x_perm, const float* s_row, int64_t rows_cap,
                                       const int32_t* offsets, int N, const void* w13q,
                                       const float* w13_scale, int d, int I, void* h,
                                       uint32_t* status, cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    CUtensorMap mr, mw, mt;
    if (!make_tma_map_2d_u8(&mr, x_perm, static_cast<uint64_t>(rows_cap), d, HALF_M)) return cudaErrorInvalidValue;
    if (!make_tma_map_2d_u8(&mw, w13q, static_cast<uint64_t>(N) * 2 * I, d, HALF_M)) return cudaErrorInvalidValue;
    if (!make_tma_map_2d_u8(&mt, x_perm, static_cast<uint64_t>(rows_cap), d, TOK_BOX)) return cudaErrorInvalidValue;
    PairArgs a = swiglu_args(rows_cap, offsets, N, d, I, h, status);
    a.row_scale = s_row;
    a.w_scale = w13_scale;
    return launch_pair<MODE_SWIGLU, true>(mr, mw, mt, a, pair_grid(di), st);
}

namespace {

PairArgs down_args(int64_t rows_cap, const int32_t* offsets, int N, int d, int I, void* y,
                   uint32_t* status) {
    PairArgs a{};
    a.offsets = offsets;
    a.out = static_cast<__nv_bfloat16*>(y);
    a.status = status;
    a.wait_ns = wait_limit_ns();
    a.clock_probe = clock_probe() ? clock_probe() + 4 : nullptr;
    a.tile_ctr = reinterpret_cast<int*>(status + 32);
    a.abort_kstep = debug_abort_kstep();
    a.rows_cap = rows_cap;
    a.ldo = d;
    a.n_groups = N;
    a.kdim = I;
    a.n_out = d;
    // 256 output features per accumulator; wide row tiles (512 features, both accumulators) when
    // d is a multiple of 512
    a.tile_cols = 2 * HALF_M;
    a.wide = d % (4 * HALF_M) == 0 ? 1 : 0;
    a.ntiles = a.wide ? d / (4 * HALF_M) : (d + 2 * HALF_M - 1) / (2 * HALF_M);
    a.b_group_rows = d;
    a.up_off = 0;
    a.s_tiles = (d + 2 * HALF_M - 1) / (2 * HALF_M);
    a.cold_rows = 128;
    a.rem_rows = 128;
    a.dbl = d % (4 * HALF_M) == 0 ? 1 : 0;
    return a;
}

}  // namespace

cudaError_t launch_grouped_down(const void* h, int64_t rows_cap, const int32_t* offsets, int N,
                                const void* w2, int d, int I, void* y, uint32_t* status,
                                cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    CUtensorMap mr, mw, mt;
    if (!make_tma_map_2d(&mr, h, static_cast<uint64_t>(rows_cap), I, HALF_M)) return cudaErrorInvalidValue;
    if (!make_tma_map_2d(&mw, w2, static_cast<uint64_t>(N) * d, I, HALF_M)) return cudaErrorInvalidValue;
    if (!make_tma_map_2d(&mt, h, static_cast<uint64_t>(rows_cap), I, TOK_BOX)) return cudaErrorInvalidValue;
    const PairArgs a = down_args(rows_cap, offsets, N, d, I, y, status);
    return launch_pair<MODE_DOWN, false>(mr, mw, mt, a, pair_grid(di), st);
}

cudaError_t launch_grouped_down_e4m3(const void* hq, const float* s_h, int64_t rows_cap,
                                     const int32_t* offsets, int N, const void* w2q,
                                     const float* w2_scale, int d, int I, void* y, uint32_t* status,
                                     cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    CUtensorMap mr, mw, mt;
    if (!make_tma_map_2d_u8(&mr, hq, static_cast<uint64_t>(rows_cap), I, HALF_M)) return cudaErrorInvalidValue;
    if (!make_tma_map_2d_u8(&mw, w2q, static_cast<uint64_t>(N) * d, I, HALF_M)) return cudaErrorInvalidValue;
    if (!make_tma_map_2d_u8(&mt, hq, static_cast<uint64_t>(rows_cap), I, TOK_BOX)) return cudaErrorInvalidValue;
    PairArgs a = down_args(rows_cap, offsets, N, d, I, y, status);
    a.row_scale = s_h;
    a.w_scale = w2_scale;
    return launch_pair<MODE_DOWN, true>(mr, mw, mt, a, pair_grid(di), st);
}

}  // namespace lcmoe
