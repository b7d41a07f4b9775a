// common.cuh -- device helpers and internal launcher declarations of libmoezero.
//
// sm_100a only: mbarriers, TMA bulk-tensor loads, tcgen05 (5th-generation tensor core) MMA with
// TMEM accumulators, written as inline PTX. No CUTLASS/CuTe code is used.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/lc_moe.h"

namespace lcmoe {

// ------------------------------------------------------------------------------ small utils --

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bits) {
    if (status) atomicOr(status, bits);
}

// ---------------------------------------------------------------------------------- mbarrier --

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// try_wait with cluster-scope acquire: the phase may have been completed by a release of the
// peer CTA, whose earlier writes into this CTA's shared memory then become visible
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// 32-bit store to a shared::cluster address (possibly in the peer CTA)
__device__ __forceinline__ void st_shared_cluster_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with parity `parity` of `bar`. Gives up (returns false) when the
// CTA-wide abort flag is raised by another role, or after `limit_ns`, in which case it raises the
// abort flag itself and records LC_MOE_DEV_WAIT_TIMEOUT.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                          volatile int* abort_flag, uint32_t* status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            set_status(status, LC_MOE_DEV_WAIT_TIMEOUT);
            return false;
        }
    }
}

// bounded wait with cluster-scope acquire (the phase was completed by the peer CTA's release)
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                                  volatile int* abort_flag, uint32_t* status) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            set_status(status, LC_MOE_DEV_WAIT_TIMEOUT);
            return false;
        }
    }
}

// ------------------------------------------------------------------------ bulk async copies --

// Contiguous copy global -> shared of `bytes` (multiple of 16, both addresses 16-byte aligned),
// completion counted on the mbarrier `bar` (no multicast).
__device__ __forceinline__ void bulk_load_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// Contiguous copy shared -> global, tracked by this thread's bulk groups.
__device__ __forceinline__ void bulk_store_s2g(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(dst), "r"(smem_u32(src)), "r"(bytes)
                 : "memory");
}
// Order this thread's view of shared memory (including copies it waited for) before later
// async-proxy accesses (bulk copies, TMA, tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's bulk groups are still reading their shared memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until at most N of this thread's bulk groups are still in flight.
template <int N>
__device__ __forceinline__ void bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------------------------- TMA --

// 2-D tiled bulk-tensor load global -> shared, completion counted on `bar` (no multicast).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ----------------------------------------------------------------------------------- tcgen05 --

// TMEM allocation: whole warp, result (lane 0 / base column) written to shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile stored with the 128-byte swizzle:
// rows of 64 bf16 (128 B), 8-row swizzle atoms of 1024 B stacked contiguously (stride-dimension
// byte offset 1024). The leading-dimension offset is unused for swizzled K-major layouts.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);  // start address >> 4, bits [0,14)
    d |= static_cast<uint64_t>(1u) << 16;                 // leading byte offset (16 B) >> 4
    d |= static_cast<uint64_t>(1024u >> 4) << 32;         // stride byte offset >> 4
    d |= static_cast<uint64_t>(1u) << 46;                 // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2u) << 61;                 // swizzle mode: 128 B
    return d;
}

// Instruction descriptor, kind::f16: A and B bf16, K-major; D fp32; shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4)                                   // D format: f32
           | (1u << 7)                                 // A format: bf16
           | (1u << 10)                                // B format: bf16
           | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Instruction descriptor, kind::f8f6f4: A and B E4M3 (format code 0), K-major; D fp32; M x N.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
    return (1u << 4)                                   // D format: f32
           | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]^T, one 128 x N x 16 step, issued by a single thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
        "}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives lane (base + i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------- CTA pairs (cta_group::2) ----

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// shared::cluster address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// arrive on an mbarrier given by its shared::cluster address (possibly in the peer CTA)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// 2-D tiled TMA load of a CTA pair: the data lands in this CTA's shared memory, the completed
// bytes are counted on the mbarrier at `bar_cluster` (the pair leader's), with an L2 policy.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int32_t c0, int32_t c1, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// D[tmem] (+)= A * B^T over a CTA pair: M = 256 (128 rows of A in each CTA), B split along N
// between the two CTAs; issued by one thread of the pair leader.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n"
        "}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// As umma_bf16_pair with E4M3 operands: one 256 x N x 32 step (32 bytes of K per operand row).
__device__ __forceinline__ void umma_e4m3_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n"
        "}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the mbarrier at the same offset in every CTA of `cta_mask` when every tcgen05
// operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}

// ------------------------------------------------------------------------ bf16 pack helpers --

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------------------- internal launchers (host side) --

struct DevInfo {
    int sm_count;
    int ok_sm100;
};

// Host-side set-up that must run once per device before a kernel's first launch there (kernel
// attributes, symbol addresses). run() calls `fn` on the current device until one call succeeds:
// concurrent first callers on any host thread are serialised by the mutex and later callers see
// the release-stored flag without locking; a failed attempt is returned to its caller and tried
// again by the next call instead of being remembered.
class PerDeviceOnce {
  public:
    static constexpr int kMaxDevices = 64;
    template <class F>
    cudaError_t run(F&& fn) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        if (done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
        std::lock_guard<std::mutex> lock(mu_);
        if (done_[dev].load(std::memory_order_relaxed)) return cudaSuccess;
        e = fn(dev);
        if (e == cudaSuccess) done_[dev].store(true, std::memory_order_release);
        return e;
    }

  private:
    std::mutex mu_;
    std::atomic<bool> done_[kMaxDevices] = {};
};
// Per-device cached properties of the current device (returns nullptr on a CUDA error).
const DevInfo* current_device_info();

uint64_t wait_limit_ns();
// Device buffer of the grouped GEMMs' clock probe (lc_moe_set_clock_probe), or nullptr.
unsigned long long* clock_probe();

// Row-major bf16 matrix [rows, cols] as a TMA map with 64 x box_rows boxes and the 128-byte swizzle.
bool make_tma_map_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows);
// Same for a row-major byte matrix (E4M3 codes) [rows, cols]: boxes of 128 bytes x box_rows.
bool make_tma_map_2d_u8(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows);

// Router GEMM: logits[T, E] fp32 = x[T, d] * wr[E, d]^T.
cudaError_t launch_router_gemm(const void* x, const void* wr, float* logits, int T, int d, int E,
                               uint32_t* status, cudaStream_t st);

// Grouped GEMM 1 (CTA pairs): h[rows, I] = silu(X Wg^T) * (X Wu^T) per expert group.
cudaError_t launch_grouped_swiglu(const void* x_perm, int64_t rows_cap, const int32_t* offsets,
                                  int N, const void* w13, int d, int I, void* h, uint32_t* status,
                                  cudaStream_t st);

// Grouped GEMM 2 (CTA pairs): y[rows, d] = h Wd^T per expert group.
cudaError_t launch_grouped_down(const void* h, int64_t rows_cap, const int32_t* offsets, int N,
                                const void* w2, int d, int I, void* y, uint32_t* status,
                                cudaStream_t st);

cudaError_t launch_topk(const float* logits, const float* bias, int T, int E, int K, int32_t* idx,
                        float* gate, int32_t* counts, uint32_t* status, cudaStream_t st);

cudaError_t launch_hist(const int32_t* idx, int64_t n, int n_bins, int32_t* counts,
                        uint32_t* status, cudaStream_t st);

cudaError_t launch_bias_update(float* bias, int32_t* counts, int E, int64_t T_all, int N, int K,
                               int K_e, float mu, int reset, cudaStream_t st);

// Scratch of the grouping step: two [nblk, N] int32 tables.
size_t permute_scratch_bytes(int T, int N);
cudaError_t launch_permute(const int32_t* idx, int T, int K, int N, int E, int32_t* offsets,
                           int32_t* row_token, int32_t* pair_row, int32_t* scratch,
                           uint32_t* status, cudaStream_t st);
cudaError_t launch_gather(const void* x, int T, int d, int K, const int32_t* pair_row,
                          void* x_perm, uint32_t* status, cudaStream_t st);
// Row gather of E4M3 token rows (d bytes each) with their scales: x_perm[pair_row[t,k]] = xq[t],
// s_row[pair_row[t,k]] = sx[t].
cudaError_t launch_gather_e4m3(const void* xq, const float* sx, int T, int d, int K,
                               const int32_t* pair_row, void* x_perm, float* s_row, uint32_t* status,
                               cudaStream_t st);

// Row-wise E4M3 quantisation of a bf16 matrix [R, C] (C % 8 == 0): scale[r] = amax / 448
// (1 for an all-zero row), dst[r, c] = E4M3(src[r, c] / scale[r]) (round to nearest even,
// saturating at 448). With rows_dev, only the first min(R, *rows_dev) rows (a count on the
// device, e.g. offsets[N]) are quantised.
cudaError_t launch_quantize_rows_e4m3(const void* src, int64_t R, int C, void* dst, float* scale,
                                      cudaStream_t st, const int32_t* rows_dev = nullptr);

// Grouped GEMM 1 on E4M3 operands: rows x_perm [rows_cap, d] (codes) with row scales s_row,
// W13 codes [N, 2I, d] with one scale per weight row; the SwiGLU epilogue applies both scales.
// Grouped GEMM 2 on E4M3 operands: hq [rows_cap, I] codes with row scales s_h, W2 codes
// [N, d, I] with one scale per weight row (output feature).
cudaError_t launch_grouped_down_e4m3(const void* hq, const float* s_h, int64_t rows_cap,
                                     const int32_t* offsets, int N, const void* w2q,
                                     const float* w2_scale, int d, int I, void* y, uint32_t* status,
                                     cudaStream_t st);

cudaError_t launch_grouped_swiglu_e4m3(const void* x_perm, const float* s_row, int64_t rows_cap,
                                       const int32_t* offsets, int N, const void* w13q,
                                       const float* w13_scale, int d, int I, void* h,
                                       uint32_t* status, cudaStream_t st);
// Grouping with its tables in a file-scope device array (no caller workspace).
bool permute_noalloc_fits(int T, int N);
cudaError_t launch_permute_noalloc(const int32_t* idx, int T, int K, int N, int E, int32_t* offsets,
                                   int32_t* row_token, int32_t* pair_row, uint32_t* status,
                                   cudaStream_t st);

cudaError_t launch_combine(const void* x, const void* y, const float* gate,
                           const int32_t* pair_row, int T, int d, int K, void* out,
                           cudaStream_t st);

cudaError_t launch_wait_check(uint32_t* status, uint64_t limit_ns, cudaStream_t st);

// Expert parallelism: expert-major permutation of rows received source-major (cnt [G, n_local],
// G * n_local <= 2048), and a row copy through an index map (gather or scatter).
cudaError_t launch_regroup_plan(const int32_t* cnt, int G, int n_local, int32_t* perm, int64_t m_cap,
                                int32_t* offsets, uint32_t* status, cudaStream_t st);
cudaError_t launch_copy_rows(const void* src, void* dst, const int32_t* map, int64_t n, int row_bytes,
                             int scatter, uint32_t* status, cudaStream_t st);

}  // namespace lcmoe
