// nm_api.cu -- status strings, the device error word and library metadata.
#include <cuda_runtime.h>
#include <stdint.h>

#include "nm_common.cuh"

namespace nm {
__device__ uint32_t g_error_word = 0;
__device__ uint64_t g_wait_limit_ns = WAIT_LIMIT_NS;
__device__ int g_test_withhold_flag_cluster = -1;
__device__ const WinTable g_wintab = WinTable();
}  // namespace nm

extern "C" nm_status nm_test_set_wait_limit_ns(unsigned long long ns) {
    const uint64_t v = ns ? static_cast<uint64_t>(ns) : nm::WAIT_LIMIT_NS;
    if (v > nm::WAIT_LIMIT_NS) return NM_ERR_SHAPE;
    return cudaMemcpyToSymbol(nm::g_wait_limit_ns, &v, sizeof(v)) == cudaSuccess ? NM_OK : NM_ERR_CUDA;
}

extern "C" nm_status nm_test_withhold_stream_k_flag(int cluster) {
    if (cluster < -1) return NM_ERR_SHAPE;
    return cudaMemcpyToSymbol(nm::g_test_withhold_flag_cluster, &cluster, sizeof(cluster)) == cudaSuccess
               ? NM_OK
               : NM_ERR_CUDA;
}

extern "C" const char *nm_status_string(int status) {
    switch (status) {
        case NM_OK: return "NM_OK";
        case NM_ERR_NULL: return "NM_ERR_NULL: a required pointer is NULL";
        case NM_ERR_SHAPE: return "NM_ERR_SHAPE: invalid or too large size / leading dimension";
        case NM_ERR_ALIGN: return "NM_ERR_ALIGN: pointer not 16-byte aligned or ld not a multiple of 8";
        case NM_ERR_UNSUPPORTED: return "NM_ERR_UNSUPPORTED: n:m pattern not supported by this call";
        case NM_ERR_WORKSPACE: return "NM_ERR_WORKSPACE: workspace or packed buffer too small";
        case NM_ERR_CUDA: return "NM_ERR_CUDA: a CUDA call failed";
        case NM_ERR_TIMEOUT: return "NM_ERR_TIMEOUT: a device-side barrier wait gave up";
        case NM_ERR_DEVICE: return "NM_ERR_DEVICE: a device-side consistency check failed";
        case NM_ERR_TOO_LARGE: return "NM_ERR_TOO_LARGE: problem exceeds the static scratch of an allocation-free call";
        default: return "unknown nm_status";
    }
}

extern "C" int nm_version(void) { return (1 << 16) | 0; }

extern "C" nm_status nm_check_device_error(void *stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return NM_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpyFromSymbol(&word, nm::g_error_word, sizeof(word)) != cudaSuccess) return NM_ERR_CUDA;
    if (word != 0) {
        const uint32_t zero = 0;
        if (cudaMemcpyToSymbol(nm::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return NM_ERR_CUDA;
    }
    if (word & nm::ERRBIT_TIMEOUT) return NM_ERR_TIMEOUT;
    if (word & nm::ERRBIT_DEVICE) return NM_ERR_DEVICE;
    return NM_OK;
}
