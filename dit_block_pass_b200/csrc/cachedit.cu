// cachedit.cu -- Cache-DiT residual-difference check, one pass over HBM.
//
// The LMSYS report summary at news.cocoloop.cn ("minimax-h3-sglang-h200"),
// section "Só com três camadas de aceleração
// somadas chega-se a 6 vezes", Cache-DiT paragraph: cached results are reused
// between neighbouring denoising steps when a residual-difference threshold
// allows it (0.04 conservative, 0.08 in the more aggressive stride mode).
// The check is the relative L1 difference of two residual tensors.
//
// Design: a partial-sum kernel on a (G, B) grid streams prev and cur once,
// 32 bytes per load when the rows allow it; G is a few device-fulls of CTAs
// (more than fit at once, which let the scheduler interleave them);
// thread sums are fp32 per 8- or 16-element vector (|cur - prev| of two bf16
// values is exact in fp32 unless their exponents are more than 16 apart) and
// fp64 above that.  Each CTA reduces with a fixed butterfly and writes its fp64
// pair to the workspace as part[g][b][2].  A one-CTA-per-sample kernel then
// adds the G pairs in a fixed order and takes the decision in fp64.  There
// are no floating-point atomics, so the result is identical run to run.
#include <math.h>

#include <mutex>

#include "common.cuh"

namespace dit {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;
constexpr int kSlotCap = 2048;  // partial-sum slots per sample in a workspace
constexpr int kWaves = 4;       // partial CTAs per sample: this many device-fulls

// Sum of |c - p| and |p| over the 8 (or 16) bf16 values of a vector pair,
// in fp32.
__device__ __forceinline__ void absdiff_sums(const uint4& pv, const uint4& cv, float& sn,
                                             float& sd) {
    float fp[8], fc[8];
    unpack8(pv, fp);
    unpack8(cv, fc);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        sn += fabsf(fc[i] - fp[i]);
        sd += fabsf(fp[i]);
    }
}

template <int E>
struct CacheVec;
template <>
struct CacheVec<8> {
    using T = uint4;
    static __device__ __forceinline__ T load(const T* p) { return ld_stream(p); }
    static __device__ __forceinline__ void sums(const T& p, const T& c, float& sn, float& sd) {
        absdiff_sums(p, c, sn, sd);
    }
};
template <>
struct CacheVec<16> {
    using T = u32x8;
    static __device__ __forceinline__ T load(const T* p) { return ld_stream256(p); }
    static __device__ __forceinline__ void sums(const T& p, const T& c, float& sn, float& sd) {
        absdiff_sums(make_uint4(p.w[0], p.w[1], p.w[2], p.w[3]),
                     make_uint4(c.w[0], c.w[1], c.w[2], c.w[3]), sn, sd);
        absdiff_sums(make_uint4(p.w[4], p.w[5], p.w[6], p.w[7]),
                     make_uint4(c.w[4], c.w[5], c.w[6], c.w[7]), sn, sd);
    }
};

// Grid (G, B): CTA g of sample b sums vectors g*T + t + k*G*T of the
// sample (T threads) and writes its fp64 pair to part[g][b][2].
template <int E>
__global__ void __launch_bounds__(kThreads)
cachedit_partials_kernel(const void* __restrict__ prev_, const void* __restrict__ cur_,
                         int64_t nvs, double* __restrict__ part, int B) {
    using V = CacheVec<E>;
    using T = typename V::T;
    const int g = blockIdx.x, b = blockIdx.y, G = gridDim.x;
    const T* P = static_cast<const T*>(prev_) + static_cast<int64_t>(b) * nvs;
    const T* C = static_cast<const T*>(cur_) + static_cast<int64_t>(b) * nvs;
    const int64_t step = static_cast<int64_t>(G) * kThreads;
    double acc_n = 0.0, acc_d = 0.0;
    for (int64_t v = static_cast<int64_t>(g) * kThreads + threadIdx.x; v < nvs;
         v += kUnroll * step) {
        T pv[kUnroll], cv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (v + u * step < nvs) {
                pv[u] = V::load(P + v + u * step);
                cv[u] = V::load(C + v + u * step);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (v + u * step < nvs) {
                float sn = 0.0f, sd = 0.0f;
                V::sums(pv[u], cv[u], sn, sd);
                acc_n += static_cast<double>(sn);
                acc_d += static_cast<double>(sd);
            }
        }
    }
    acc_n = warp_sum(acc_n);
    acc_d = warp_sum(acc_d);
    __shared__ double sh[2][kThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        sh[0][warp] = acc_n;
        sh[1][warp] = acc_d;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double n = 0.0, d = 0.0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) {
            n += sh[0][w];
            d += sh[1][w];
        }
        double* out = part + (static_cast<int64_t>(g) * B + b) * 2;
        out[0] = n;
        out[1] = d;
    }
}

// One CTA of kThreads per sample: thread t adds partial pairs t, t + T, ...
// (part[r][b][2]) in order, then the CTA combines the thread sums through a
// fixed butterfly and a fixed warp order, and thread 0 writes the sums and/or
// the decision.  The order depends only on R, so equal inputs give equal bits.
__global__ void __launch_bounds__(kThreads)
cachedit_finalize_kernel(const double* __restrict__ part, int R, int B, double threshold,
                         double* sums_out, double* rel_out, uint8_t* reuse_out) {
    const int b = blockIdx.x;
    double n = 0.0, d = 0.0;
    for (int r = threadIdx.x; r < R; r += kThreads) {
        n += part[(static_cast<int64_t>(r) * B + b) * 2];
        d += part[(static_cast<int64_t>(r) * B + b) * 2 + 1];
    }
    n = warp_sum(n);
    d = warp_sum(d);
    __shared__ double sh[2][kThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        sh[0][warp] = n;
        sh[1][warp] = d;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        n = 0.0;
        d = 0.0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) {
            n += sh[0][w];
            d += sh[1][w];
        }
        if (sums_out) {
            sums_out[2 * b] = n;
            sums_out[2 * b + 1] = d;
        }
        if (rel_out) {
            double rel;
            if (d == 0.0) rel = (n == 0.0) ? 0.0 : INFINITY;
            else rel = n / d;
            rel_out[b] = rel;
            reuse_out[b] = rel < threshold ? 1 : 0;
        }
    }
}

// Partial-sum slots per sample: `waves` times the CTAs that fit on the
// device at once (more CTAs than fit lets the scheduler interleave them),
// at most kSlotCap, at least 1.
int partial_slots(int B, int64_t nvs, int waves) {
    const int sms = device_sm_count();
    if (sms <= 0) return 0;
    const int occ =
        occupancy(reinterpret_cast<const void*>(cachedit_partials_kernel<8>), kThreads, 0);
    int64_t g = static_cast<int64_t>(sms) * occ * waves / B;
    const int64_t need = (nvs + kThreads - 1) / kThreads;
    if (g > need) g = need;
    if (g > kSlotCap) g = kSlotCap;
    if (g < 1) g = 1;
    return static_cast<int>(g);
}

int check_inputs(const uint16_t* prev, const uint16_t* cur, int B, int64_t N, int D) {
    if (B < 1 || N < 0 || D <= 0) return DIT_ERR_SHAPE;
    if (B > 65535 || N > (INT64_MAX / 8) / D / B) return DIT_ERR_SHAPE;
    if (D % 8) return DIT_ERR_ALIGN;
    if (N == 0) return DIT_OK;  // nothing is read: prev and cur may be NULL
    if (!prev || !cur) return DIT_ERR_NULL;
    if (!aligned16(prev) || !aligned16(cur)) return DIT_ERR_ALIGN;
    return DIT_OK;
}

int run_partials(const uint16_t* prev, const uint16_t* cur, int B, int64_t N, int D,
                 void* workspace, size_t workspace_bytes, cudaStream_t stream, int* slots) {
    if (!workspace || !aligned16(workspace)) return DIT_ERR_WORKSPACE;
    if (workspace_bytes < cachedit_workspace_bytes(B, N, D)) return DIT_ERR_WORKSPACE;
    // 32-byte vectors when every sample's rows allow them
    const bool wide = D % 16 == 0 && aligned32(prev) && aligned32(cur);
    const int64_t nvs = N * D / (wide ? 16 : 8);
    const int G = partial_slots(B, nvs, kWaves);
    if (G < 1) return DIT_ERR_LAUNCH;
    dim3 grid(static_cast<unsigned>(G), static_cast<unsigned>(B));
    if (wide)
        cachedit_partials_kernel<16><<<grid, kThreads, 0, stream>>>(
            prev, cur, nvs, static_cast<double*>(workspace), B);
    else
        cachedit_partials_kernel<8><<<grid, kThreads, 0, stream>>>(
            prev, cur, nvs, static_cast<double*>(workspace), B);
    *slots = G;
    return launch_status();
}

}  // namespace
}  // namespace dit

extern "C" size_t cachedit_workspace_bytes(int B, int64_t N, int D) {
    (void)N;
    (void)D;
    if (B < 1) return 0;
    return static_cast<size_t>(B) * dit::kSlotCap * 2 * sizeof(double);
}

extern "C" int cachedit_residual_diff(const uint16_t* prev, const uint16_t* cur, int B, int64_t N,
                                      int D, double threshold, double* rel_out,
                                      uint8_t* reuse_out, void* workspace,
                                      size_t workspace_bytes, void* stream) {
    using namespace dit;
    int st = check_inputs(prev, cur, B, N, D);
    if (st) return st;
    if (!rel_out || !reuse_out) return DIT_ERR_NULL;
    if (isnan(threshold)) return DIT_ERR_VALUE;
    int G = 0;
    if ((st = run_partials(prev, cur, B, N, D, workspace, workspace_bytes, as_stream(stream), &G)))
        return st;
    cachedit_finalize_kernel<<<B, kThreads, 0, as_stream(stream)>>>(
        static_cast<const double*>(workspace), G, B, threshold, nullptr, rel_out, reuse_out);
    return launch_status();
}

extern "C" int cachedit_residual_sums(const uint16_t* prev, const uint16_t* cur, int B, int64_t N,
                                      int D, double* sums_out, void* workspace,
                                      size_t workspace_bytes, void* stream) {
    using namespace dit;
    int st = check_inputs(prev, cur, B, N, D);
    if (st) return st;
    if (!sums_out) return DIT_ERR_NULL;
    int G = 0;
    if ((st = run_partials(prev, cur, B, N, D, workspace, workspace_bytes, as_stream(stream), &G)))
        return st;
    cachedit_finalize_kernel<<<B, kThreads, 0, as_stream(stream)>>>(
        static_cast<const double*>(workspace), G, B, 0.0, sums_out, nullptr, nullptr);
    return launch_status();
}

extern "C" int cachedit_decide(const double* sums, int R, int B, double threshold,
                               double* rel_out, uint8_t* reuse_out, void* stream) {
    using namespace dit;
    if (!sums || !rel_out || !reuse_out) return DIT_ERR_NULL;
    if (R < 1 || B < 1 || B > 65535) return DIT_ERR_SHAPE;
    if (reinterpret_cast<uintptr_t>(sums) % 8) return DIT_ERR_ALIGN;
    if (isnan(threshold)) return DIT_ERR_VALUE;
    cachedit_finalize_kernel<<<B, kThreads, 0, dit::as_stream(stream)>>>(sums, R, B, threshold, nullptr,
                                                                  rel_out, reuse_out);
    return launch_status();
}

// ---------------------------------------------------------------------------
// Cache-DiT check without a caller-provided workspace.
//
// Some callers cannot call cudaMalloc or hand this library a scratch buffer:
// for example a plugin inside a serving engine that owns every byte of device
// memory through its own pool and forbids raw allocations, or a caller on a
// latency-critical path that cannot afford the device-wide synchronisation a
// fresh cudaMalloc can cause.  For them the partial sums live in a fixed
// array in this library's device memory: kStaticPairs (sum, sum) pairs, 64 KB,
// which every GPU that loads the library holds until the process exits.
//
// Host code must not pass the array's name to a kernel (on the host it is a
// stand-in, not a device address); the device address comes from
// cudaGetSymbolAddress with that device current.  It is looked up again on
// every call made outside stream capture (a cudaDeviceReset reloads the
// module at a new address), and a call made while its stream is capturing
// uses the address the last uncaptured call on that device found.
namespace dit {
namespace {

constexpr int kStaticMaxSamples = 64;
constexpr int kStaticPairs = 4096;
static __device__ __align__(256) double g_cachedit_scratch[kStaticPairs * 2];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
double* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device: looked up
// when the stream is not capturing, else the one cached by an earlier call
// (NULL if there was none).
double* scratch_address(cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    const bool capturing =
        cudaStreamIsCapturing(stream, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!capturing) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_cachedit_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = static_cast<double*>(p);
    }
    return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace dit

extern "C" int cachedit_residual_diff_noalloc(const uint16_t* prev, const uint16_t* cur, int B,
                                              int64_t N, int D, double threshold,
                                              double* rel_out, uint8_t* reuse_out,
                                              void* stream) {
    using namespace dit;
    int st = check_inputs(prev, cur, B, N, D);
    if (st) return st;
    if (B > kStaticMaxSamples) return DIT_ERR_SHAPE;
    if (!rel_out || !reuse_out) return DIT_ERR_NULL;
    if (isnan(threshold)) return DIT_ERR_VALUE;
    double* scratch = scratch_address(as_stream(stream));
    if (!scratch) return DIT_ERR_LAUNCH;
    const int64_t nvs = N * D / 8;
    const int G = partial_slots(B, nvs, 1);
    if (G < 1) return DIT_ERR_LAUNCH;
    if (static_cast<int64_t>(G) * B > kStaticPairs) return DIT_ERR_WORKSPACE;
    // Every slot the finalize kernel reads is written by the partials kernel
    // of the same call, so the array needs no clearing between calls.
    dim3 grid(static_cast<unsigned>(G), static_cast<unsigned>(B));
    cachedit_partials_kernel<8><<<grid, kThreads, 0, as_stream(stream)>>>(prev, cur, nvs, scratch,
                                                                         B);
    if ((st = launch_status())) return st;
    cachedit_finalize_kernel<<<B, kThreads, 0, as_stream(stream)>>>(scratch, G, B, threshold, nullptr,
                                                              rel_out, reuse_out);
    return launch_status();
}
