// dart_common.cuh -- small device helpers shared by the DART kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dart.h"

namespace dart {

// Device status word bits (latched by kernels, read by dart_sync_status).
enum : int {
    kStatusTimeout = 1,   // a bounded wait gave up
    kStatusDevice = 2,    // bad device-side state (decode counters / cache full)
};

// The status word lives in dart_abi.cu (one per device); kernels receive its
// device address and set bits with atomicOr.
__device__ __forceinline__ void flag_status(int* status, int bits) { atomicOr(status, bits); }

// ---------------------------------------------------------------------------
// element conversion
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float to_f(float v) { return v; }
    static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

template <typename T> __device__ __forceinline__ float ldf(const T* p) { return Elem<T>::to_f(*p); }

// 16-byte vector of T unpacked to floats: 4 floats or 8 bf16.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int kN = 4;
    static __device__ __forceinline__ void load(const float* p, float* out) {
        float4 v = *reinterpret_cast<const float4*>(p);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
    static __device__ __forceinline__ void load_nc(const float* p, float* out) {
        float4 v = __ldg(reinterpret_cast<const float4*>(p));
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
    static __device__ __forceinline__ void store(float* p, const float* in) {
        *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int kN = 8;
    static __device__ __forceinline__ void unpack(uint4 v, float* out) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* out) {
        unpack(*reinterpret_cast<const uint4*>(p), out);
    }
    static __device__ __forceinline__ void load_nc(const __nv_bfloat16* p, float* out) {
        unpack(__ldg(reinterpret_cast<const uint4*>(p)), out);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* in) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

// Streaming 16-byte load that does not allocate in L1 (read-once data).
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// log2(e): the softmax runs in base 2 on scores pre-multiplied by it.
constexpr float kLog2e = 1.4426950408889634f;

}  // namespace dart

// Host-side launch helpers implemented per kernel family.
namespace dart {
// B and C are shared by groups of heads (Mamba-2 ngroups): with G groups
// (G divides H) they are [B, L, G, N] and head h reads group h / (H / G);
// G = 1 is the [B, L, N] layout shared by all heads.
__host__ __device__ __forceinline__ int group_of(int h, int H, int G) { return h / (H / G); }

struct ScanArgs {
    int B, L, H, P, N, S, G;
    const void* x; const float* dt; const float* A; const void* Bm; const void* Cm;
    const float* init_state;
    float* y; void* dH; float* states; float* asum;  // asum: [B,H,C] workspace
    void* hin;    // tensor-core path: bf16 state entering each chunk [B,H,C,N,P] (workspace)
    float* decay; // tensor-core path: per-token decay terms, 3 x [B,H,C,S] fp32 (workspace)
    int* status;  // device status word
};
struct SmaArgs {
    int B, L, H, P, N, S, G;
    const void* Q; const void* E; const void* Cm; const void* dH;
    float g; const float* y_ssd; float* out;
    int* status;  // device status word
    // Decayed-memory variant (both set) or raw memories (both null): the
    // base-2 exponent of memory c's decay at token t of chunk k is
    // la2[b,h,t] + gpre[b,h,k] - gpre[b,h,c+1] (see sma_decay.cu).
    const float* la2;     // [B,H,C*S] fp32
    const double* gpre;   // [B,H,C] fp64
};
struct DecodeArgs {
    int B, H, P, N, S, G, cmax, nsplit;
    const void* x; const float* dt; const float* A; const void* Bm; const void* Cm;
    const void* Q; const void* E; float g;
    float* state; float* dHcur; void* cache; int* nchunks; int* pos; float* y;
    float* part;  // [B,H,nsplit,2+2P] workspace
    int* status;  // device status word
    // Decayed-memory variant (null: raw memories): [B,H,cmax] fp32, the
    // log-decay sum_{r=e(c)+1}^{t-1} dt_r A_h each cached memory carries.
    float* memlog;
    // E4M3 cache (null: the cache holds dtype values): cache holds E4M3 codes
    // [B,H,cmax,N,P] and cexp the row exponents [B,H,cmax,N] (value = code 2^k).
    signed char* cexp;
};

// Counts one kernel launch (see dart_launch_count).
void count_launches(int n);

// Launches `kernel` so that it may start while the previous launch on the
// stream finishes (programmatic dependent launch); the kernel must call
// sm100::griddep_wait() before touching global memory.  cluster_x > 1
// launches clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             int cluster_x, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (cluster_x > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)cluster_x;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)na;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

cudaError_t launch_ssd_scan(const ScanArgs& a, dart_dtype dt, cudaStream_t st);
cudaError_t launch_sma(const SmaArgs& a, dart_dtype dt, cudaStream_t st);
cudaError_t launch_decode(const DecodeArgs& a, dart_dtype dt, cudaStream_t st);
bool ssd_scan_supported(int N, int P, int S, dart_dtype dt);
bool ssd_scan_tc_applicable(int N, int P, int S, dart_dtype dt);
cudaError_t launch_ssd_scan_tc(const ScanArgs& a, cudaStream_t st);
bool sma_supported(int N, int P, int S, dart_dtype dt);
bool sma_tc_applicable(int N, int P, int S, dart_dtype dt);
cudaError_t launch_sma_tc(const SmaArgs& a, cudaStream_t st);
// Decay terms of the decayed-memory SMA from dt [B,L,H] and A [H] into la2 and
// gpre (layouts as in SmaArgs); two launches.
cudaError_t launch_sma_decay_terms(int B, int L, int H, int S, const float* dt, const float* A,
                                   float* la2, double* gpre, cudaStream_t st);
size_t sma_decay_workspace_bytes(int B, int L, int H, int S);
const char* sma_impl_name(int N, int P, int S, dart_dtype dt);
bool decode_supported(int N, int P, int S, dart_dtype dt);
int decode_num_splits(int B, int H, int cmax);
// Largest cache capacity the decode entries accept (memories per sequence):
// 2^20 memories is 2^28 tokens of context at S = 256.
constexpr int kDecodeMaxCmax = 1 << 20;
bool decode_e4m3_supported(int N, int P);
cudaError_t launch_decode_e4m3(const DecodeArgs& a, dart_dtype dt, cudaStream_t st);
// selftest.cu: one bounded wait on an mbarrier nothing arrives on.
cudaError_t launch_wait_drill(int* status, unsigned long long limit_ns, cudaStream_t st);
// dH [B,H,C,N,P] (dtype) memories 0..nmem-1 -> E4M3 codes and row exponents
// in cache slots 0..nmem-1 ([B,H,cmax,N,P] / [B,H,cmax,N]); one launch.
cudaError_t launch_cache_quantize_e4m3(int B, int H, int C, int N, int P, int nmem, int cmax, const void* dH,
                                       dart_dtype dt, unsigned char* cache, signed char* cexp, cudaStream_t st);
// memlog[b,h,c] = sum_{r=(c+1)S}^{L-1} dt[b,r,h] A[h] for c < L / S (one launch).
cudaError_t launch_decode_memlog_init(int B, int L, int H, int S, int cmax, const float* dt, const float* A,
                                      float* memlog, cudaStream_t st);

// dart_decode_step_noalloc: size of the library-owned static scratch, and its
// device address on the current device (set up on the first call per device).
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
cudaError_t noalloc_scratch(void** out);
}  // namespace dart
