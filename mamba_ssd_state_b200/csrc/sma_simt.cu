// sma_simt.cu -- state-memory attention on CUDA cores (fp32 path and the
// shapes the tensor-core kernel does not cover).
//
// Per token t of chunk k(t) and every chunk memory c < k(t) (Pith review of
// DART, "Core claim" / "What carries the argument"; SMA Eqs. (5)-(10)):
//   u = Q_t^T dH[c] (P),  v = C_t^T dH[c] (P),  s = u . E_t / sqrt(N)
// which equals Q_t . (dH[c] E_t) / sqrt(N) -- the key read out of the memory by
// contracting its value axis -- by associativity.  An online softmax over c
// accumulates o_t; the epilogue writes y_ssd + g * o_t (or o_t alone).
// In the decayed-memory variant (referee comment 3 on Eq. (8)) memory c is
// scaled by w = exp(sum_{r=e(c)+1}^{t} dt_r A_h) before use: the score becomes
// w s and the value w v (terms from sma_decay.cu).
//
// One block = 64 query tokens of one (b, h), all in the same chunk; 4 threads
// per token, each owning P/4 output columns.  The memory dH[c] is staged in
// shared memory once per block and shared by the 64 tokens.
#include "dart_common.cuh"

namespace dart {
namespace {

constexpr int kThreads = 256;
constexpr int kTQ = 64;

template <typename T, int N, int P>
__global__ void __launch_bounds__(kThreads) sma_simt_kernel(SmaArgs a) {
    constexpr int PT = P / 4;
    constexpr int NS = N + 4;          // padded row stride, keeps float4 alignment
    const int S = a.S, C = (a.L + S - 1) / S;
    const int t0 = blockIdx.x * kTQ;   // first token of the tile
    const int h = blockIdx.y, b = blockIdx.z;
    const int k = t0 / S;              // chunk of every token in the tile
    extern __shared__ __align__(16) float sm[];
    float* Qs = sm;                    // [kTQ][NS], pre-scaled by log2(e)/sqrt(N)
    float* Cs = Qs + kTQ * NS;         // [kTQ][NS]
    float* Ms = Cs + kTQ * NS;         // [N][P]
    const T* Q = static_cast<const T*>(a.Q);
    const T* E = static_cast<const T*>(a.E);
    const T* Cm = static_cast<const T*>(a.Cm);
    const T* dH = static_cast<const T*>(a.dH);
    const float qscale = kLog2e * rsqrtf((float)N);

    const int tl = threadIdx.x / 4, pg = threadIdx.x % 4;
    const int t = t0 + tl;
    const bool live = t < a.L;         // rows past the end of a partial last chunk only help load tiles
    float o[PT], e[PT];
#pragma unroll
    for (int j = 0; j < PT; ++j) {
        o[j] = 0.f;
        e[j] = live ? ldf(E + (((size_t)b * a.L + t) * a.H + h) * P + pg * PT + j) : 0.f;
    }
    float mrun = -INFINITY, lrun = 0.f;
    const bool decayed = a.la2 != nullptr;
    const size_t bh = (size_t)b * a.H + h;
    // decayed variant: t's in-chunk log2 prefix and the chunk prefix at k
    const float la_t = decayed && live ? a.la2[bh * C * S + t] : 0.f;
    const double g_k = decayed && k > 0 ? a.gpre[bh * C + k] : 0.0;

    if (k > 0) {
        for (int i = threadIdx.x; i < kTQ * N; i += blockDim.x) {
            const int r = i / N, n = i % N;
            const bool in = t0 + r < a.L;
            const size_t tok = (size_t)b * a.L + t0 + r;
            Qs[r * NS + n] = in ? qscale * ldf(Q + (tok * a.H + h) * N + n) : 0.f;
            Cs[r * NS + n] = in ? ldf(Cm + (tok * a.G + group_of(h, a.H, a.G)) * N + n) : 0.f;
        }
        const T* mem = dH + ((size_t)b * a.H + h) * (size_t)C * N * P;
        for (int c = 0; c < k; ++c) {
            __syncthreads();
            for (int i = threadIdx.x; i < N * P; i += blockDim.x) Ms[i] = ldf(mem + (size_t)c * N * P + i);
            __syncthreads();
            float u[PT], v[PT];
#pragma unroll
            for (int j = 0; j < PT; ++j) u[j] = v[j] = 0.f;
            for (int n = 0; n < N; n += 4) {
                const float4 q4 = *reinterpret_cast<const float4*>(Qs + tl * NS + n);
                const float4 c4 = *reinterpret_cast<const float4*>(Cs + tl * NS + n);
                const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
                const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) {
                    const float* row = Ms + (n + nn) * P + pg * PT;
#pragma unroll
                    for (int j = 0; j < PT; ++j) {
                        u[j] = fmaf(qv[nn], row[j], u[j]);
                        v[j] = fmaf(cv[nn], row[j], v[j]);
                    }
                }
            }
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < PT; ++j) s = fmaf(u[j], e[j], s);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            float wd = 1.f;   // decay of memory c at token t (1 for raw memories)
            if (decayed) {
                wd = exp2f(la_t + (float)(g_k - a.gpre[bh * C + c + 1]));
                s *= wd;
            }
            const float mnew = fmaxf(mrun, s);
            const float alpha = exp2f(mrun - mnew);
            const float w = exp2f(s - mnew);
            lrun = lrun * alpha + w;
            const float wv = w * wd;
#pragma unroll
            for (int j = 0; j < PT; ++j) o[j] = fmaf(o[j], alpha, wv * v[j]);
            mrun = mnew;
        }
    }
    if (!live) return;
    const float inv = k > 0 ? 1.f / lrun : 0.f;
    const size_t row = (((size_t)b * a.L + t) * a.H + h) * P + pg * PT;
#pragma unroll
    for (int j = 0; j < PT; ++j) {
        const float oj = o[j] * inv;
        a.out[row + j] = a.y_ssd ? fmaf(a.g, oj, a.y_ssd[row + j]) : oj;
    }
}

template <typename T, int N, int P>
cudaError_t run(const SmaArgs& a, cudaStream_t st) {
    const size_t smem = sizeof(float) * (2 * kTQ * (N + 4) + N * P);
    auto k = sma_simt_kernel<T, N, P>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<dim3((a.L + kTQ - 1) / kTQ, a.H, a.B), kThreads, smem, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launches(1);
    return cudaSuccess;
}

}  // namespace

bool sma_supported(int N, int P, int S, dart_dtype) {
    const bool np = (N == 16 && P == 16) || (N == 64 && P == 64) || (N == 128 && P == 64);
    return np && (S == 64 || S == 128 || S == 256);
}

const char* sma_impl_name(int N, int P, int S, dart_dtype dt) {
    return sma_tc_applicable(N, P, S, dt) ? "sma_tcgen05" : "sma_simt";
}

cudaError_t launch_sma(const SmaArgs& a, dart_dtype dt, cudaStream_t st) {
    if (sma_tc_applicable(a.N, a.P, a.S, dt)) return launch_sma_tc(a, st);
#define DART_SMA_CASE(NN, PP)                                                       \
    if (a.N == NN && a.P == PP)                                                     \
        return dt == DART_F32 ? run<float, NN, PP>(a, st) : run<__nv_bfloat16, NN, PP>(a, st);
    DART_SMA_CASE(16, 16)
    DART_SMA_CASE(64, 64)
    DART_SMA_CASE(128, 64)
#undef DART_SMA_CASE
    return cudaErrorInvalidValue;
}

}  // namespace dart
