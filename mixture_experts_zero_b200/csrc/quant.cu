// quant.cu -- row-wise E4M3 quantisation for the FP8 experts.
//
// The LongCat-Flash llm-wiki entity page, section 5 (inference and deployment), deploys the model
// with FP8 weights; the scheme used here gives every row (a token row of x, or one output feature
// of the gate/up weights) one fp32 scale:
//   s_r = max_c |x_rc| / 448   (one IEEE division; 1 for an all-zero row)
//   q_rc = E4M3(x_rc / s_r)    (one IEEE division, then round to nearest even, saturating at 448)
// so that x_rc ~ s_r * q_rc. One warp per row: a first pass takes the row's absolute maximum, a
// second pass (from L1/L2) converts 8 bf16 values per lane and step into 8 E4M3 bytes.
#include "common.cuh"

namespace lcmoe {

namespace {

constexpr int QUANT_THREADS = 256;

// Two fp32 values to two E4M3 codes: lo in the low byte, hi in the high byte.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__global__ void __launch_bounds__(QUANT_THREADS)
    quantize_rows_kernel(const uint4* __restrict__ src, int64_t R, int c8, uint2* __restrict__ dst,
                         float* __restrict__ scale, const int32_t* __restrict__ rows_dev) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (rows_dev) {
        const int64_t rd = *rows_dev;
        if (rd < R) R = rd < 0 ? 0 : rd;
    }
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (QUANT_THREADS / 32);
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * (QUANT_THREADS / 32) + warp; r < R;
         r += warps_total) {
        const uint4* row = src + r * c8;
        float amax = 0.0f;
        for (int c = lane; c < c8; c += 32) {
            const uint4 v = __ldg(row + c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                amax = fmaxf(amax, fmaxf(fabsf(bf16lo(w[j])), fabsf(bf16hi(w[j]))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        if (lane == 0) scale[r] = s;
        uint2* out = dst + r * c8;
        for (int c = lane; c < c8; c += 32) {
            const uint4 v = __ldg(row + c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint16_t q[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                q[j] = e4m3x2(__fdiv_rn(bf16lo(w[j]), s), __fdiv_rn(bf16hi(w[j]), s));
            out[c] = make_uint2(static_cast<uint32_t>(q[0]) | (static_cast<uint32_t>(q[1]) << 16),
                                static_cast<uint32_t>(q[2]) | (static_cast<uint32_t>(q[3]) << 16));
        }
    }
}

}  // namespace

cudaError_t launch_quantize_rows_e4m3(const void* src, int64_t R, int C, void* dst, float* scale,
                                      cudaStream_t st, const int32_t* rows_dev) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    if (R == 0) return cudaSuccess;
    const int warps = QUANT_THREADS / 32;
    int64_t blocks = (R + warps - 1) / warps;
    if (blocks > static_cast<int64_t>(di->sm_count) * 16) blocks = static_cast<int64_t>(di->sm_count) * 16;
    quantize_rows_kernel<<<static_cast<int>(blocks), QUANT_THREADS, 0, st>>>(
        static_cast<const uint4*>(src), R, C / 8, static_cast<uint2*>(dst), scale, rows_dev);
    return cudaGetLastError();
}

}  // namespace lcmoe
