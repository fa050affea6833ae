// rb_abi.cu -- small C-ABI helpers shared by every entry point: version,
// status names, sizes, device queries.
#include "rbw_internal.cuh"

#include <atomic>

namespace rbw {

int num_sms()
{
    static std::atomic<int> cache[64];         // per device, 0 = not yet queried
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

bool device_is_sm100()
{
    static std::atomic<int> cache[64];         // per device: 0 unknown, 1 yes, 2 no
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (dev >= 0 && dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c) return c == 1;
    }
    int major = 0;
    const bool ok = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess && major == 10;
    if (dev >= 0 && dev < 64) cache[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
    return ok;
}

}  // namespace rbw

extern "C" int rb_version(void) { return 100; }   // 0.1.0

extern "C" const char* rb_status_string(int status)
{
    switch (status) {
        case RB_OK: return "RB_OK";
        case RB_ERR_ARG: return "RB_ERR_ARG";
        case RB_ERR_SHAPE: return "RB_ERR_SHAPE";
        case RB_ERR_ALIGN: return "RB_ERR_ALIGN";
        case RB_ERR_WORKSPACE: return "RB_ERR_WORKSPACE";
        case RB_ERR_UNSUPPORTED: return "RB_ERR_UNSUPPORTED";
        case RB_ERR_CUDA: return "RB_ERR_CUDA";
        default: return "RB_ERR_UNKNOWN";
    }
}

extern "C" size_t rb_packed_words(int n_out, int k_in, int k_planes)
{
    if (n_out < 1 || k_in < 32 || k_in % 32 != 0 || k_planes < 1 || k_planes > 8) return 0;
    return (size_t)k_planes * (size_t)rbw::num_slices(k_in) * (size_t)rbw::num_row_tiles(n_out) * 256u;
}
