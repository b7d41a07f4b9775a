// route.cu -- routing of the MoE layer with zero-computation experts, and the expert-bias
// controller (LongCat-Flash llm-wiki entity page, section 2.1; softmax gate: section 2.3.2).
//
//   topk      : per token, s = softmax(z) over all E = N + Z experts; key_i = s_i + b_i;
//               the K largest keys in descending order (equal keys: lower index first), found by
//               K rounds of a warp-wide max over each lane's best untaken key, then a warp-wide
//               min over the indices of the lanes holding that key;
//               gate_r = s_sel[r] / (s_sel[0] + ... + s_sel[K-1]); optional histogram of picks.
//   hist      : T_i, the number of picks of each expert (the T_i of the bias-update equation).
//   bias      : b_i += mu * (K_e/(K N) - T_i/(K T_all)) for all E experts.
//
// Routing decisions are integers decided in fp32, so the fp32 steps are fixed exactly:
//   exp: Cody-Waite reduction (Cody & Waite, Software Manual for the Elementary Functions, 1980)
//        u = n ln2 + r, n = rint(u log2e), ln2 split into a 16-fraction-bit head and a tail,
//        then e^r by its degree-7 Taylor polynomial (coefficients 1/k!) in Horner form with
//        fused multiply-adds, times 2^n; inputs below -86 give 0;
//   sum: lane l of the warp adds e_l, e_{l+32}, ... in order from +0, then the lanes combine by
//        a butterfly over xor distances 16, 8, 4, 2, 1 (both operands of every add are the same
//        pair of values on the two lanes, so all lanes end with identical bits);
//   every other step is one IEEE round-to-nearest operation (__f*_rn intrinsics, no contraction).
#include "common.cuh"

namespace lcmoe {

namespace {

// fp32 constants of the exp above, from ln 2 and 1/k!. Branch-free: the argument is clamped to
// [-86, 88] for the arithmetic and the result is replaced by 0 below -86, +inf above 88 and the
// argument itself when it is NaN (the same values as the specification's early returns).
__device__ __forceinline__ float exp_spec(float u) {
    const float LOG2E = 0x1.715476p+0f;     // 1/ln 2, rounded to fp32
    const float LN2_HI = 0x1.62e4p-1f;      // ln 2 rounded to 16 fraction bits (exact)
    const float LN2_LO = 0x1.7f7d1cp-20f;   // ln 2 - LN2_HI, rounded to fp32
    const float uc = fminf(fmaxf(u, -86.0f), 88.0f);
    const float n = rintf(__fmul_rn(uc, LOG2E));
    float r = __fmaf_rn(-n, LN2_HI, uc);
    r = __fmaf_rn(-n, LN2_LO, r);
    float p = 0x1.a01a02p-13f;              // 1/7!
    p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);   // 1/6!
    p = __fmaf_rn(p, r, 0x1.111112p-7f);    // 1/5!
    p = __fmaf_rn(p, r, 0x1.555556p-5f);    // 1/4!
    p = __fmaf_rn(p, r, 0x1.555556p-3f);    // 1/3!
    p = __fmaf_rn(p, r, 0.5f);              // 1/2!
    p = __fmaf_rn(p, r, 1.0f);              // 1/1!
    p = __fmaf_rn(p, r, 1.0f);              // 1/0!
    const float scale = __int_as_float((static_cast<int>(n) + 127) << 23);  // 2^n, normal
    float e = __fmul_rn(p, scale);
    e = (u < -86.0f) ? 0.0f : e;
    e = (u > 88.0f) ? __int_as_float(0x7f800000) : e;
    return (u != u) ? u : e;
}

constexpr int TOPK_THREADS = 256;  // 8 warps, one token per warp at a time

template <int VPL>
__global__ void __launch_bounds__(TOPK_THREADS)
    topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E,
                int K, int32_t* __restrict__ idx, float* __restrict__ gate,
                int32_t* __restrict__ counts, uint32_t* __restrict__ status) {
    extern __shared__ int32_t smem_i[];
    int32_t* s_hist = smem_i;                                   // [E]
    float* s_bias = reinterpret_cast<float*>(smem_i + E);      // [E]
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    float* s_score = s_bias + E + warp * E;                     // [8][E]: this warp's token scores
    const bool do_hist = counts != nullptr;
    for (int i = threadIdx.x; i < E; i += TOPK_THREADS) {
        s_hist[i] = 0;
        s_bias[i] = bias[i];
    }
    __syncthreads();

    const int warps_total = gridDim.x * (TOPK_THREADS / 32);
    // up to 32 values per lane (E <= 1024), the next token's logits are loaded while the current
    // one is processed; above that the registers are needed for the current token
    constexpr bool PREFETCH = VPL <= 32;
    float vn[PREFETCH ? VPL : 1];
    auto load = [&](int tt, float* dst) {
        const float* zt = logits + static_cast<int64_t>(tt) * E;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int i = lane + 32 * j;
            dst[j] = (tt < T && i < E) ? __ldcs(zt + i) : __int_as_float(0xff800000);
        }
    };
    if (PREFETCH) load(blockIdx.x * (TOPK_THREADS / 32) + warp, vn);
    for (int t = blockIdx.x * (TOPK_THREADS / 32) + warp; t < T; t += warps_total) {
        float v[VPL];
        if (PREFETCH) {
#pragma unroll
            for (int j = 0; j < VPL; ++j) v[j] = vn[PREFETCH ? j : 0];
            load(t + warps_total, vn);
        } else {
            load(t, v);
        }
        float m = __int_as_float(0xff800000);  // -inf
#pragma unroll
        for (int j = 0; j < VPL; ++j)
            m = (v[j] > m) ? v[j] : m;  // a NaN logit is skipped here, and poisons the sum below
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float other = __shfl_xor_sync(0xffffffffu, m, o);
            m = (other > m) ? other : m;
        }
        // e_i = EXP(z_i - m); lane partial sums in index order
        float part = 0.0f;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int i = lane + 32 * j;
            if (i < E) {
                v[j] = exp_spec(__fsub_rn(v[j], m));
                part = __fadd_rn(part, v[j]);
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) part = __fadd_rn(part, __shfl_xor_sync(0xffffffffu, part, o));
        const float S = part;
        // scores s_i = e_i / S and keys s_i + b_i, the keys as order-preserving unsigned integers
        // (no key is -0: scores are >= +0, and +0 + -0 rounds to +0; 0 is below every key)
        uint32_t ku[VPL];
        bool nan_key = false;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int i = lane + 32 * j;
            ku[j] = 0;
            if (i < E) {
                v[j] = __fdiv_rn(v[j], S);
                s_score[i] = v[j];
                const float key = __fadd_rn(v[j], s_bias[i]);
                nan_key |= (key != key);
                const uint32_t kb = __float_as_uint(key);
                ku[j] = (kb & 0x80000000u) ? ~kb : (kb | 0x80000000u);
            }
        }
        if (__any_sync(0xffffffffu, nan_key)) {
            if (lane == 0) set_status(status, LC_MOE_DEV_NAN_KEY);
            if (lane < K) {
                idx[static_cast<int64_t>(t) * K + lane] = lane;
                gate[static_cast<int64_t>(t) * K + lane] = __int_as_float(0x7fc00000);
                if (do_hist) atomicAdd(&s_hist[lane], 1);
            }
            continue;
        }
        // K rounds of warp arg-max over (key, index); each lane keeps its best three untaken keys
        // (with their indices) and rescans only when all three are taken. The scores are kept in
        // this warp's shared-memory row, read back for the K winners only.
        uint64_t taken = 0;
        uint32_t k1 = 0, k2 = 0, k3 = 0;
        int i1 = 0x7fffffff, i2 = 0x7fffffff, i3 = 0x7fffffff;
        auto top3 = [&]() {
            k1 = k2 = k3 = 0;
            i1 = i2 = i3 = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const int i = lane + 32 * j;
                const uint32_t kj = ((taken >> j) & 1ull) ? 0u : ku[j];  // ku = 0 (past E) never wins
                if (kj > k3) {
                    if (kj > k2) {
                        k3 = k2; i3 = i2;
                        if (kj > k1) {
                            k2 = k1; i2 = i1;
                            k1 = kj; i1 = i;
                        } else {
                            k2 = kj; i2 = i;
                        }
                    } else {
                        k3 = kj; i3 = i;
                    }
                }
            }
        };
        top3();
        int my_idx = 0;
        for (int r = 0; r < K; ++r) {
            const uint32_t m = __reduce_max_sync(0xffffffffu, k1);
            const int w = __reduce_min_sync(0xffffffffu, k1 == m ? static_cast<uint32_t>(i1) : 0x7fffffffu);
            if (lane == r) my_idx = w;
            if ((w & 31) == lane) {
                taken |= 1ull << (w >> 5);
                k1 = k2; i1 = i2;
                k2 = k3; i2 = i3;
                k3 = 0; i3 = 0x7fffffff;
                if (k1 == 0) top3();
            }
        }
        __syncwarp();
        const float my_s = lane < K ? s_score[my_idx] : 0.0f;
        // renormalise over the K chosen, summing in rank order
        float Q = 0.0f;
        for (int r = 0; r < K; ++r) Q = __fadd_rn(Q, __shfl_sync(0xffffffffu, my_s, r));
        if (lane < K) {
            idx[static_cast<int64_t>(t) * K + lane] = my_idx;
            gate[static_cast<int64_t>(t) * K + lane] = __fdiv_rn(my_s, Q);
            if (do_hist) atomicAdd(&s_hist[my_idx], 1);
        }
    }
    if (do_hist) {
        __syncthreads();
        for (int i = threadIdx.x; i < E; i += TOPK_THREADS) {
            const int c = s_hist[i];
            if (c) atomicAdd(&counts[i], c);
        }
    }
}

template <int VPL>
cudaError_t launch_topk_t(const float* logits, const float* bias, int T, int E, int K,
                          int32_t* idx, float* gate, int32_t* counts, uint32_t* status,
                          cudaStream_t st, int sm_count) {
    const int warps = TOPK_THREADS / 32;
    int blocks = (T + warps - 1) / warps;
    const int cap = sm_count * 4;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    // histogram, biases and one score row per warp: 80 KB at E = 2048
    const size_t smem = (2 + warps) * static_cast<size_t>(E) * sizeof(int32_t);
    static PerDeviceOnce setup;
    const cudaError_t e = setup.run([](int) {
        return cudaFuncSetAttribute(topk_kernel<VPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>((2 + TOPK_THREADS / 32) * 32 * VPL * sizeof(int32_t)));
    });
    if (e != cudaSuccess) return e;
    topk_kernel<VPL><<<blocks, TOPK_THREADS, smem, st>>>(logits, bias, T, E, K, idx, gate, counts,
                                                          status);
    return cudaGetLastError();
}

constexpr int HIST_THREADS = 512;
constexpr int HIST_UNROLL = 4;

__global__ void __launch_bounds__(HIST_THREADS)
    hist_kernel(const int32_t* __restrict__ idx, int64_t n, int n_bins, int32_t* __restrict__ counts,
                uint32_t* __restrict__ status) {
    extern __shared__ int32_t s_hist[];
    for (int i = threadIdx.x; i < n_bins; i += HIST_THREADS) s_hist[i] = 0;
    __syncthreads();
    bool bad = false;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * HIST_THREADS;
    const int64_t n4 = n / 4;
    const int4* idx4 = reinterpret_cast<const int4*>(idx);
    // HIST_UNROLL 16-byte loads in flight per thread before their shared-memory atomics
    for (int64_t p0 = static_cast<int64_t>(blockIdx.x) * HIST_THREADS + threadIdx.x; p0 < n4;
         p0 += HIST_UNROLL * stride) {
        int4 q[HIST_UNROLL];
#pragma unroll
        for (int u = 0; u < HIST_UNROLL; ++u) {
            const int64_t p = p0 + u * stride;
            q[u] = p < n4 ? __ldg(idx4 + p) : make_int4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < HIST_UNROLL; ++u) {
            if (p0 + u * stride >= n4) break;
            const int vals[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (vals[j] >= 0 && vals[j] < n_bins) atomicAdd(&s_hist[vals[j]], 1);
                else bad = true;
            }
        }
    }
    for (int64_t p = n4 * 4 + static_cast<int64_t>(blockIdx.x) * HIST_THREADS + threadIdx.x; p < n; p += stride) {
        const int v = idx[p];
        if (v >= 0 && v < n_bins) atomicAdd(&s_hist[v], 1);
        else bad = true;
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) set_status(status, LC_MOE_DEV_IDX_RANGE);
    for (int i = threadIdx.x; i < n_bins; i += HIST_THREADS) {
        const int c = s_hist[i];
        if (c) atomicAdd(&counts[i], c);
    }
}

__global__ void bias_update_kernel(float* __restrict__ bias, int32_t* __restrict__ counts, int E,
                                   long long T_all, int N, int K, int K_e, float mu, int reset) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= E) return;
    const float kn = __fmul_rn(static_cast<float>(K), static_cast<float>(N));
    const float a = __fdiv_rn(static_cast<float>(K_e), kn);
    const float kt = __fmul_rn(static_cast<float>(K), __ll2float_rn(T_all));
    const float c = __fdiv_rn(__int2float_rn(counts[i]), kt);
    const float delta = __fmul_rn(mu, __fsub_rn(a, c));
    bias[i] = __fadd_rn(bias[i], delta);
    if (reset) counts[i] = 0;
}

}  // namespace

cudaError_t launch_topk(const float* logits, const float* bias, int T, int E, int K, int32_t* idx,
                        float* gate, int32_t* counts, uint32_t* status, cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    const int vpl = (E + 31) / 32;
    const int sm = di->sm_count;
    if (vpl <= 1) return launch_topk_t<1>(logits, bias, T, E, K, idx, gate, counts, status, st, sm);
    if (vpl <= 2) return launch_topk_t<2>(logits, bias, T, E, K, idx, gate, counts, status, st, sm);
    if (vpl <= 4) return launch_topk_t<4>(logits, bias, T, E, K, idx, gate, counts, status, st, sm);
    if (vpl <= 8) return launch_topk_t<8>(logits, bias, T, E, K, idx, gate, counts, status, st, sm);
    if (vpl <= 12) return launch_topk_t<12>(logits, bias, T, E, K, idx, gate, counts, status, st, sm);
    if (vpl <= 16) return launch_topk_t<16>(logits, bias, T, E, K, idx, gate, counts, status, st, sm);
    if (vpl <= 24) return launch_topk_t<24>(logits, bias, T, E, K, idx, gate, counts, status, st, sm);
    if (vpl <= 32) return launch_topk_t<32>(logits, bias, T, E, K, idx, gate, counts, status, st, sm);
    if (vpl <= 48) return launch_topk_t<48>(logits, bias, T, E, K, idx, gate, counts, status, st, sm);
    return launch_topk_t<64>(logits, bias, T, E, K, idx, gate, counts, status, st, sm);
}

cudaError_t launch_hist(const int32_t* idx, int64_t n, int n_bins, int32_t* counts,
                        uint32_t* status, cudaStream_t st) {
    const DevInfo* di = current_device_info();
    if (!di) return cudaErrorUnknown;
    int64_t blocks = (n / 4 + HIST_THREADS - 1) / HIST_THREADS;
    if (blocks > di->sm_count * 2) blocks = di->sm_count * 2;
    if (blocks < 1) blocks = 1;
    hist_kernel<<<static_cast<int>(blocks), HIST_THREADS, static_cast<size_t>(n_bins) * 4, st>>>(
        idx, n, n_bins, counts, status);
    return cudaGetLastError();
}

cudaError_t launch_bias_update(float* bias, int32_t* counts, int E, int64_t T_all, int N, int K,
                               int K_e, float mu, int reset, cudaStream_t st) {
    const int threads = 256;
    const int blocks = (E + threads - 1) / threads;
    bias_update_kernel<<<blocks, threads, 0, st>>>(bias, counts, E, static_cast<long long>(T_all), N,
                                                   K, K_e, mu, reset);
    return cudaGetLastError();
}

}  // namespace lcmoe
