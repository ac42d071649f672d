// status.cu -- ABI version, status strings and the per-device attribute cache.
#include <mutex>
#include <unordered_map>

#include "common.cuh"

namespace dit {

namespace {
std::mutex g_mu;
std::unordered_map<int, int> g_sms;
std::unordered_map<uint64_t, int> g_occ;  // key: device, kernel, threads, smem
}  // namespace

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_sms.find(dev);
    if (it != g_sms.end()) return it->second;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms = 0;
    if (sms > 0) g_sms[dev] = sms;
    return sms;
}

int occupancy(const void* kernel, int threads, size_t smem) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    uint64_t key = (static_cast<uint64_t>(dev) << 56) ^
                   (reinterpret_cast<uintptr_t>(kernel) * 0x9E3779B97F4A7C15ull) ^
                   (static_cast<uint64_t>(threads) << 32) ^ static_cast<uint64_t>(smem);
    {
        std::lock_guard<std::mutex> lock(g_mu);
        auto it = g_occ.find(key);
        if (it != g_occ.end()) return it->second;
    }
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kernel, threads, smem) !=
            cudaSuccess || blocks < 1)
        blocks = 1;
    std::lock_guard<std::mutex> lock(g_mu);
    g_occ[key] = blocks;
    return blocks;
}

}  // namespace dit

extern "C" int dit_abi_version(void) { return 1; }

extern "C" const char* dit_status_string(int status) {
    switch (status) {
        case DIT_OK: return "ok";
        case DIT_ERR_NULL: return "a required pointer is NULL";
        case DIT_ERR_SHAPE: return "a size is out of range";
        case DIT_ERR_ALIGN: return "a pointer or row length breaks the 16-byte alignment rule";
        case DIT_ERR_DTYPE: return "unknown dtype";
        case DIT_ERR_LAUNCH: return "CUDA launch error";
        case DIT_ERR_WORKSPACE: return "workspace missing or too small";
        case DIT_ERR_OVERLAP: return "buffers overlap where they may not";
        case DIT_ERR_VALUE: return "a scalar argument is out of range";
        default: return "unknown status";
    }
}
