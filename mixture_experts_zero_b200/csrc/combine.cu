// combine.cu -- the weighted sum of the MoE equation, with the zero-computation experts fused.
//
//   out_t = sum_{r < K} g_{t,r} * v_{t,r},   v = Y[pair_row] for an FFN pick,
//                                            v = x_t          for a zero-computation pick
// (LongCat-Flash llm-wiki entity page, section 2.1: E_i(x_t) = x_t for the Z zero experts).
// One warp per token; each lane owns 8-element (16-byte) column chunks and accumulates in fp32,
// in rank order, with one fused multiply-add per pick: the zero-expert term costs one read of
// x_t per token (shared by all its zero picks) and no extra pass.
#include "common.cuh"

namespace lcmoe {

namespace {

constexpr int COMBINE_THREADS = 256;

// Loads in flight per lane: two 16-byte column chunks (c and c + 32) of PB picks at a time.
constexpr int PB = 4;

__device__ __forceinline__ void fma_row(float (&acc)[8], float g, const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        acc[2 * j] = __fmaf_rn(g, bf16lo(w[j]), acc[2 * j]);
        acc[2 * j + 1] = __fmaf_rn(g, bf16hi(w[j]), acc[2 * j + 1]);
    }
}

__device__ __forceinline__ uint4 pack8(const float (&acc)[8]) {
    return make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                      pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
}

// Work item: one token's row (SPLIT = false), or a (token, column block) of `span` 16-byte chunks
// (SPLIT = true, when T is too small for one warp per token to fill the GPU).
template <bool SPLIT>
__global__ void __launch_bounds__(COMBINE_THREADS)
    combine_kernel(const uint4* __restrict__ x, const uint4* __restrict__ y,
                   const float* __restrict__ gate, const int32_t* __restrict__ pair_row, int T,
                   int d8, int K, int cb, int span, uint4* __restrict__ out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (COMBINE_THREADS / 32);
    const int items = SPLIT ? T * cb : T;  // T * cb stays near the warp count of one wave
    for (int it = blockIdx.x * (COMBINE_THREADS / 32) + warp; it < items; it += warps_total) {
        const int t = SPLIT ? it / cb : it;
        const int c_begin = SPLIT ? (it - t * cb) * span : 0;
        const int c_end = SPLIT ? min(d8, c_begin + span) : d8;
        float my_g = 0.0f;
        int my_row = -1;
        if (lane < K) {
            my_g = gate[static_cast<int64_t>(t) * K + lane];
            my_row = pair_row[static_cast<int64_t>(t) * K + lane];
        }
        const bool any_zero = __any_sync(0xffffffffu, lane < K && my_row < 0);
        const uint4* xt = x + static_cast<int64_t>(t) * d8;
        for (int c0 = c_begin; c0 < c_end; c0 += 64) {  // warp-uniform trip count
            const int ca = c0 + lane, cb2 = c0 + 32 + lane;
            const bool ina = ca < c_end, inb = cb2 < c_end;
            uint4 xa = make_uint4(0, 0, 0, 0), xb = xa;
            if (any_zero) {
                if (ina) xa = __ldg(xt + ca);
                if (inb) xb = __ldg(xt + cb2);
            }
            float acc_a[8], acc_b[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc_a[j] = acc_b[j] = 0.0f;
            for (int r0 = 0; r0 < K; r0 += PB) {
                float g[PB];
                int row[PB];
                uint4 va[PB], vb[PB];
#pragma unroll
                for (int u = 0; u < PB; ++u) {
                    g[u] = __shfl_sync(0xffffffffu, my_g, (r0 + u) & 31);
                    row[u] = __shfl_sync(0xffffffffu, my_row, (r0 + u) & 31);
                }
#pragma unroll
                for (int u = 0; u < PB; ++u) {
                    const bool pick = r0 + u < K;
                    const uint4* yr = y + static_cast<int64_t>(row[u] < 0 ? 0 : row[u]) * d8;
                    va[u] = (pick && row[u] >= 0 && ina) ? __ldg(yr + ca) : xa;
                    vb[u] = (pick && row[u] >= 0 && inb) ? __ldg(yr + cb2) : xb;
                }
                // rank order: pick r0, r0 + 1, ... each one fused multiply-add per element
#pragma unroll
                for (int u = 0; u < PB; ++u) {
                    if (r0 + u < K) {
                        fma_row(acc_a, g[u], va[u]);
                        fma_row(acc_b, g[u], vb[u]);
                    }
                }
            }
            if (ina) out[static_cast<int64_t>(t) * d8 + ca] = pack8(acc_a);
            if (inb) out[static_cast<int64_t>(t) * d8 + cb2] = pack8(acc_b);
        }
    }
}

}  // namespace

cudaError_t launch_combine(const void* x, const void* y, const float* gate,
                           const int32_t* pair_row, int T, int d, int K, void* out,
                           cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    if (T == 0) return cudaSuccess;
    const int warps = COMBINE_THREADS / 32;
    const int d8 = d / 8;
    // column blocks per token: enough (token, block) items for 8 blocks of 8 warps per SM
    const int max_cb = (d8 + 63) / 64;
    int cb = (di->sm_count * 8 * warps + T - 1) / T;
    if (cb > max_cb) cb = max_cb;
    if (cb < 1) cb = 1;
    const int span = ((d8 + cb - 1) / cb + 63) / 64 * 64;
    cb = (d8 + span - 1) / span;
    const int64_t items = static_cast<int64_t>(T) * cb;
    int64_t blocks = (items + warps - 1) / warps;
    if (blocks > di->sm_count * 8) blocks = di->sm_count * 8;
    if (cb > 1)
        combine_kernel<true><<<static_cast<int>(blocks), COMBINE_THREADS, 0, st>>>(
            static_cast<const uint4*>(x), static_cast<const uint4*>(y), gate, pair_row, T, d8, K, cb, span,
            static_cast<uint4*>(out));
    else
        combine_kernel<false><<<static_cast<int>(blocks), COMBINE_THREADS, 0, st>>>(
            static_cast<const uint4*>(x), static_cast<const uint4*>(y), gate, pair_row, T, d8, K, 1, d8,
            static_cast<uint4*>(out));
    return cudaGetLastError();
}

}  // namespace lcmoe
