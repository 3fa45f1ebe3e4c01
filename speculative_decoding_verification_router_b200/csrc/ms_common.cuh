// Shared host/device helpers of libmoespec: launch with programmatic
// dependent launch, tracing hooks, device status word, bounded waits.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stdlib.h>
#include <atomic>
#include <utility>

#include "moespec.h"

namespace ms {

// ------------------------------------------------------------ kernel ids
enum KernelId : int {
    K_RMSNORM = 0,
    K_ROUTE_ROWS,
    K_ROUTE_TILED,
    K_ROUTE_CLUSTER,
    K_PERMUTE_COUNT,
    K_PERMUTE_SCATTER,
    K_FFN_PREP,
    K_GEMM1_STREAM,
    K_GEMM2_STREAM,
    K_GEMM1_TILED,
    K_GEMM2_TILED,
    K_FFN_FINISH,
    K_LM_HEAD,
    K_COMBINE,
    K_VERIFY_PARTIAL,
    K_VERIFY_FINAL,
    K_VERIFY_CLUSTER,
    K_VERIFY_KEYS,
    K_WAIT_PROBE,
    K_PACK,
    K_MTP_PREP,
    K_LAYER_FUSED,
    K_ROUTE_TC,
    K_ROUTE_SPLIT,
    K_COUNT
};
const char* kernel_name(int id);

// ------------------------------------------------------------ host side
void trace_mark(int id, cudaStream_t s, bool after);
uint64_t wait_limit_ns();
int batch_invariant();
void set_cuda_error(cudaError_t e);

// Programmatic dependent launch is on unless MOESPEC_NO_PDL=1 (a measurement
// knob: kernels are correct either way, since each waits for its predecessor).
inline int pdl_allowed() {
    static const int on = [] {
        const char* e = getenv("MOESPEC_NO_PDL");
        return (e && e[0] == '1') ? 0 : 1;
    }();
    return on;
}

// Launch `kernel` with programmatic stream serialisation allowed, so that it
// may start while the previous kernel on the stream finishes; the kernel
// itself calls grid_dep_wait() before touching dependent memory.
template <typename... KArgs, typename... Args>
inline ms_status launch(int id, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                        cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_allowed();
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    trace_mark(id, s, false);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    trace_mark(id, s, true);
    if (e != cudaSuccess) {
        set_cuda_error(e);
        return MS_ERR_CUDA;
    }
    return MS_OK;
}

// Same, launched as thread-block clusters of `cluster_x` CTAs along x.
template <typename... KArgs, typename... Args>
inline ms_status launch_cluster(int id, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                cudaStream_t s, int cluster_x, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_allowed();
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    trace_mark(id, s, false);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    trace_mark(id, s, true);
    if (e != cudaSuccess) {
        set_cuda_error(e);
        return MS_ERR_CUDA;
    }
    return MS_OK;
}

// ------------------------------------------------------------ per-device host caches
// Values the host code looks up once per device (SM count, cluster sizes,
// occupancy) and one-time function attributes (which apply to the device
// that is current when they are set).  Each cache holds one slot per device,
// filled by the first call with that device current; the slots are atomics,
// so two host threads racing on the first fill both compute the same value
// and neither reads a half-written one.
constexpr int kMaxDevices = 64;

inline int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        dev = 0;
    }
    return dev;
}

// `fill()` must return a non-zero value (0 marks an empty slot).
struct PerDevice {
    std::atomic<int> v[kMaxDevices];
    template <typename F>
    int get(F fill) {
        std::atomic<int>& slot = v[current_device()];
        int x = slot.load(std::memory_order_acquire);
        if (x == 0) {
            x = fill();
            slot.store(x, std::memory_order_release);
        }
        return x;
    }
};

inline int num_sms() {
    static PerDevice cache;
    return cache.get([] {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, current_device()) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        return n;
    });
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------ device side
// Wait for the kernel this one depends on (no-op when launched without PDL).
// Every kernel of this library calls grid_dep_launch only after its own
// grid_dep_wait, so when kernel N starts, kernel N-2 has completed and its
// writes are visible: a kernel may read what came from two or more launches
// back before its own wait, and only what its direct predecessor writes after.
__device__ __forceinline__ void grid_dep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Allow the next kernel on the stream to be scheduled.
__device__ __forceinline__ void grid_dep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Record the first device-side error into a status word (first writer wins).
__device__ __forceinline__ void report_status(int32_t* status, int32_t code) {
    if (status) atomicCAS(status, 0, code);
}

// A drain wait (the bounded wait, after a timeout, for a CTA's own loads or
// MMAs still in flight) ran out as well: recorded over any earlier status,
// since the CTA now exits with asynchronous work possibly outstanding.
__device__ __forceinline__ void drain_failed(int32_t* status, volatile int& flag) {
    if (status) atomicExch(status, MS_ERR_DRAIN_TIMEOUT);
    flag = 1;
}

// Warp-wide (value, index) argmax step: larger value wins, equal values go
// to the lower index.
__device__ __forceinline__ void argmax_merge(float& v, int& i, float v2, int i2) {
    if (v2 > v || (v2 == v && i2 < i)) {
        v = v2;
        i = i2;
    }
}

__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float v2 = __shfl_xor_sync(0xffffffffu, v, o);
        int i2 = __shfl_xor_sync(0xffffffffu, i, o);
        argmax_merge(v, i, v2, i2);
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---- thread-block clusters: distributed shared memory and the cluster barrier
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Store v into the same shared-memory variable of CTA `rank` of this cluster.
__device__ __forceinline__ void st_cluster_f32(const void* local, uint32_t rank, float v) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local));
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_s32(const void* local, uint32_t rank, int v) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local));
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(ra), "r"(v) : "memory");
}
// Every thread of every CTA of the cluster must reach this; it orders the
// stores above before the loads after it, cluster-wide.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The value of the same shared-memory int in the other CTA of a pair
// (after a cluster barrier that orders its last store).
__device__ __forceinline__ int peer_flag(const volatile int* local) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(const_cast<int*>(local)));
    uint32_t ra;
    int v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(cluster_rank() ^ 1u));
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(ra) : "memory");
    return v;
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

}  // namespace ms
