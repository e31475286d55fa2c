// Sticky per-device status word that the kernels set when a device-side check
// fails (bad block id, bad slot, bad context length, copy-wait timeout), plus
// the error-reporting entry points of the C ABI.
#include <mutex>

#include "common.cuh"

namespace {

__device__ int g_status_word;  // one per device that loads the library

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {};
std::mutex g_status_mu;
thread_local int t_last_cuda_error = 0;

}  // namespace

namespace pkv {

void record_cuda_error(cudaError_t e) { t_last_cuda_error = (int)e; }

int* status_word_for_current_device()
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        record_cuda_error(e == cudaSuccess ? cudaErrorInvalidDevice : e);
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_status_word);
        if (e != cudaSuccess) {
            record_cuda_error(e);
            return nullptr;
        }
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    return g_status_ptr[dev];
}

}  // namespace pkv

namespace {

// One warp waits, with the kernels' own bounded wait, on an mbarrier that
// nothing ever arrives on.  The wait gives up after limit_ns and records
// PKV_DEV_WAIT_TIMEOUT, exactly as a decode kernel would if its copies
// never landed.
__global__ void wait_timeout_kernel(uint64_t limit_ns, int* status, int* gave_up)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        pkv::mbar_init(&bar, 1);
        pkv::fence_mbar_init();
    }
    __syncwarp();
    if (!pkv::mbar_wait(&bar, 0, limit_ns)) {
        if (threadIdx.x == 0) {
            pkv::raise_flag(status, PKV_DEV_WAIT_TIMEOUT);
            if (gave_up) *gave_up = 1;
        }
    }
}

}  // namespace

extern "C" {

int pkv_debug_wait_timeout(int64_t limit_ns, void* stream)
{
    if (limit_ns < 0 || limit_ns > 1000000000ll) return PKV_ERR_INVALID_ARG;
    int* status = pkv::status_word_for_current_device();
    if (!status) return PKV_ERR_CUDA;
    wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_ns, status, nullptr);
    return pkv::check_launch();
}


int pkv_device_status(int32_t device, int32_t* flags_out, int32_t clear)
{
    if (!flags_out) return PKV_ERR_INVALID_ARG;
    int prev = 0;
    cudaError_t e = cudaGetDevice(&prev);
    if (e != cudaSuccess) {
        pkv::record_cuda_error(e);
        return PKV_ERR_CUDA;
    }
    if ((e = cudaSetDevice(device)) != cudaSuccess) {
        pkv::record_cuda_error(e);
        return PKV_ERR_INVALID_ARG;
    }
    int rc = PKV_OK;
    int* word = pkv::status_word_for_current_device();
    int value = 0;
    if (!word) {
        rc = PKV_ERR_CUDA;
    } else if ((e = cudaDeviceSynchronize()) != cudaSuccess ||
               (e = cudaMemcpy(&value, word, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess) {
        pkv::record_cuda_error(e);
        rc = PKV_ERR_CUDA;
    } else if (clear && (e = cudaMemset(word, 0, sizeof(int))) != cudaSuccess) {
        pkv::record_cuda_error(e);
        rc = PKV_ERR_CUDA;
    }
    *flags_out = value;
    cudaSetDevice(prev);
    return rc;
}

int pkv_last_cuda_error(void) { return t_last_cuda_error; }

const char* pkv_status_string(int status)
{
    switch (status) {
        case PKV_OK: return "ok";
        case PKV_ERR_INVALID_ARG: return "invalid argument";
        case PKV_ERR_UNSUPPORTED: return "unsupported dtype or shape";
        case PKV_ERR_CUDA: return "CUDA error (see pkv_last_cuda_error)";
        case PKV_ERR_OUT_OF_BLOCKS: return "out of free blocks";
        case PKV_ERR_BAD_BLOCK: return "bad block id";
        case PKV_ERR_DEVICE: return "device-side check failed";
        case PKV_ERR_SCRATCH_LIMIT: return "batch needs more scratch than the fixed no-alloc array";
        case PKV_ERR_HOST_MEMORY: return "host memory could not be allocated";
        default: return "unknown status";
    }
}

}  // extern "C"
