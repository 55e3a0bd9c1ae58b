// libindexcache_probe.so (include/indexcache_probe.h): measurement and test
// aids kept out of the method's library.  The K/V row gather of the
// sparse-attention kernel alone, to measure the random-row gather ceiling
// that bounds attention when K/V sit in L2; and one bounded device wait that
// runs out, for the failure-detection test.  Not part of the method.  Links
// against libindexcache.so (error messages, the context's error word).
#include "../../../include/indexcache_probe.h"
#include "../ic_device.cuh"
#include "../ic_internal.h"

namespace ic {

constexpr int kProbeWarps = 4;
constexpr int kProbeStages = 2;             // chunks in flight per warp
constexpr int kProbeChunk = 16 * 256 * 2;   // 16 rows of K and of V (d = 128)
constexpr int kProbeIdxSlots = 2 * kProbeStages;
constexpr int kProbeSmem = kProbeWarps * (kProbeStages * kProbeChunk + kProbeIdxSlots * 64);

// Each warp walks its CTA's rows' chunks (chunk j of a row belongs to warp
// j mod kProbeWarps) with kProbeStages chunks of K/V rows in flight.  The
// 16 index slots of a chunk reach a per-warp shared ring two stages ahead
// of their gather (16-byte cp.async in the group of an earlier chunk), so
// issuing a gather never waits on an index load: only the gathers' own
// latency and bandwidth are measured.
__global__ void __launch_bounds__(kProbeWarps * 32)
    k_probe_gather(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
                   const int32_t* __restrict__ idx, int rows, int k, unsigned* __restrict__ sink) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t base = smem_u32(smem) + warp * kProbeStages * kProbeChunk;
    int32_t* iring = reinterpret_cast<int32_t*>(smem + kProbeWarps * kProbeStages * kProbeChunk) +
                     warp * kProbeIdxSlots * 16;
    const int piece = lane & 15, prow = lane >> 4;
    const int nch = k / (16 * kProbeWarps);  // chunks per warp per row
    const int nrow = blockIdx.x < rows ? (rows - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const long long total = static_cast<long long>(nrow) * nch;
    auto slots = [&](long long g) {  // the index slots of this warp's chunk g
        const int r = blockIdx.x + static_cast<int>(g / nch) * gridDim.x;
        const int c0 = (warp + static_cast<int>(g % nch) * kProbeWarps) * 16;
        return idx + static_cast<long long>(r) * k + c0;
    };
    unsigned acc = 0;
    for (long long g = 0; g < kProbeIdxSlots && g < total; ++g)
        if (lane < 16) iring[g * 16 + lane] = __ldg(slots(g) + lane);
    __syncwarp();
    auto issue = [&](long long g) {
        if (g < total) {
            const uint32_t st = base + static_cast<uint32_t>(g % kProbeStages) * kProbeChunk;
            int32_t* ir = iring + (g % kProbeIdxSlots) * 16;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int row = prow + 2 * i;
                const int s = ir[row];
                const uint32_t off = static_cast<uint32_t>(row * 256 + ((piece ^ (row & 7)) << 4));
                cp_async16(st + off, K + static_cast<long long>(s) * 128 + piece * 8, true);
                cp_async16(st + 4096 + off, V + static_cast<long long>(s) * 128 + piece * 8, true);
            }
            __syncwarp();  // every lane has read the ring slot: refill it
            const long long gn = g + kProbeIdxSlots;
            if (gn < total && lane < 4) cp_async16(smem_u32(ir + lane * 4), slots(gn) + lane * 4, true);
        }
        cp_async_commit();
    };
#pragma unroll
    for (int s = 0; s < kProbeStages; ++s) issue(s);
    for (long long g = 0; g < total; ++g) {
        cp_async_wait<kProbeStages - 1>();
        __syncwarp();
        acc += *reinterpret_cast<const volatile unsigned*>(
            smem + (warp * kProbeStages + g % kProbeStages) * kProbeChunk + lane * 4);
        __syncwarp();
        issue(g + kProbeStages);
    }
    cp_async_wait<0>();
    if (acc == 0x9e3779b9u) sink[0] = acc;  // keeps the loads observable
}

}  // namespace ic

extern "C" int ic_probe_gather(const void* K, const void* V, const int32_t* idx, int rows, int k,
                               int d, int ctas_per_sm, void* stream) {
    if (!K || !V || !idx) return ic::fail(nullptr, IC_ERR_INVALID_ARG, "probe_gather: NULL");
    if (d != 128 || k <= 0 || k % 64 != 0 || rows <= 0 || ctas_per_sm < 1 || ctas_per_sm > 3 ||
        (reinterpret_cast<uintptr_t>(idx) & 15) != 0)
        return ic::fail(nullptr, IC_ERR_UNSUPPORTED, "probe_gather: d=%d k=%d rows=%d", d, k, rows);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int smem = ic::kProbeSmem;
    cudaError_t e = cudaFuncSetAttribute(ic::k_probe_gather,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return ic::cuda_fail(nullptr, e, "probe_gather attribute");
    const int grid = sms * ctas_per_sm < rows ? sms * ctas_per_sm : rows;
    ic::k_probe_gather<<<grid, ic::kProbeWarps * 32, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16*>(K), static_cast<const __nv_bfloat16*>(V), idx, rows, k,
        nullptr);
    e = cudaGetLastError();
    if (e != cudaSuccess) return ic::cuda_fail(nullptr, e, "probe_gather launch");
    return IC_OK;
}

namespace ic {

// One bounded wait on a barrier that nothing arrives at: the library's
// bounded mbarrier wait gives up after its limit and latches the timeout code.
__global__ void k_probe_wait_timeout(int* err) {
    __shared__ uint64_t bar;
    __shared__ int abort_s;
    if (threadIdx.x == 0) {
        abort_s = 0;
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_s, err, kDevTimeoutProducer);
}

}  // namespace ic

extern "C" int ic_probe_wait_timeout(ic_ctx* ctx, void* stream) {
    if (!ctx) return ic::fail(nullptr, IC_ERR_INVALID_ARG, "probe_wait_timeout: context is NULL");
    cudaSetDevice(ctx->device);
    ic::k_probe_wait_timeout<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(ctx->dev_err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return ic::cuda_fail(ctx, e, "probe_wait_timeout launch");
    return IC_OK;
}
