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

__global__ void __launch_bounds__(COMBINE_THREADS)
    combine_kernel(const uint4* __restrict__ x, const uint4* __restrict__ y,
                   const float* __restrict__ gate, const int32_t* __restrict__ pair_row, int T,
                   int d8, int K, uint4* __restrict__ out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (COMBINE_THREADS / 32);
    for (int t = blockIdx.x * (COMBINE_THREADS / 32) + warp; t < T; t += warps_total) {
        float my_g = 0.0f;
        int my_row = -1;
        if (lane < K) {
            my_g = gate[static_cast<int64_t>(t) * K + lane];
            my_row = pair_row[static_cast<int64_t>(t) * K + lane];
        }
        const bool any_zero = __any_sync(0xffffffffu, lane < K && my_row < 0);
        const uint4* xt = x + static_cast<int64_t>(t) * d8;
        for (int c0 = 0; c0 < d8; c0 += 32) {  // warp-uniform trip count
            const int c = c0 + lane;
            const bool in = c < d8;
            uint4 xv = make_uint4(0, 0, 0, 0);
            if (in && any_zero) xv = __ldg(xt + c);
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
            for (int r = 0; r < K; ++r) {
                const float g = __shfl_sync(0xffffffffu, my_g, r);
                const int row = __shfl_sync(0xffffffffu, my_row, r);
                if (!in) continue;
                const uint4 v = (row >= 0) ? __ldg(y + static_cast<int64_t>(row) * d8 + c) : xv;
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[2 * j] = __fmaf_rn(g, bf16lo(w[j]), acc[2 * j]);
                    acc[2 * j + 1] = __fmaf_rn(g, bf16hi(w[j]), acc[2 * j + 1]);
                }
            }
            if (in)
                out[static_cast<int64_t>(t) * d8 + c] =
                    make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                               pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
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
    int blocks = (T + warps - 1) / warps;
    if (blocks > di->sm_count * 8) blocks = di->sm_count * 8;
    combine_kernel<<<blocks, COMBINE_THREADS, 0, st>>>(static_cast<const uint4*>(x),
                                                        static_cast<const uint4*>(y), gate, pair_row,
                                                        T, d / 8, K, static_cast<uint4*>(out));
    return cudaGetLastError();
}

}  // namespace lcmoe
