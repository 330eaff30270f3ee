// ssd_scan_simt.cu -- Mamba-2 SSD chunked scan that keeps the chunk memories.
//
// Three kernels, run in order on one stream (Mamba-2 SSD chunked scan, as used
// by DART: "Transformers are SSMs" SSD view, Eq. (4); Pith review of DART,
// "What carries the argument" for the retained chunk contribution dH[c]):
//
//   chunk_state   per (b, h, c): Acum_s = sum_{r=cS}^{s} dt_r A_h, then
//                 dH[c] = sum_s B_s (exp(Acum_e - Acum_s) dt_s x_s)^T.
//                 Writes dH in the input dtype, its float value into
//                 states[c] (consumed in place by state_pass), and
//                 Asum[c] = Acum_e to the workspace.
//   state_pass    per (b, h, element of N x P): states[c] = exp(Asum[c])
//                 states[c-1] + dH[c], sequential in c (in place).
//   chunk_output  per (b, h, 64-token tile): intra-chunk quadratic block
//                 sum_{s<=t} (C_t.B_s) exp(Acum_t - Acum_s) dt_s x_s plus the
//                 inter-chunk term exp(Acum_t) C_t^T states[c-1].
//
// This file is the CUDA-core path: it serves fp32 inputs (whose 1e-4
// tolerance rules out reduced-precision tensor-core inputs) and every
// (N, P, S) outside the tensor-core kernel's compiled shape.
#include "dart_common.cuh"

namespace dart {
namespace {

constexpr int kThreads = 256;

// Inclusive prefix sum of v[0..n) in shared memory, n <= blockDim.x.
__device__ void block_inclusive_scan(float* v, int n) {
    for (int off = 1; off < n; off <<= 1) {
        float add = 0.f;
        if (threadIdx.x < n && threadIdx.x >= off) add = v[threadIdx.x - off];
        __syncthreads();
        if (threadIdx.x < n) v[threadIdx.x] += add;
        __syncthreads();
    }
}

// dt of token t of batch b, head h; 0 past the end of a partial last chunk
// (no decay, no input), so the chunk's sums stop at token L-1.
__device__ __forceinline__ float dt_at(const ScanArgs& a, int b, int t, int h) {
    return t < a.L ? a.dt[((size_t)b * a.L + t) * a.H + h] : 0.f;
}

// Acum[s] for the chunk starting at token t0 of (b, h).
__device__ void load_chunk_cumsum(const ScanArgs& a, int b, int h, int t0, float* acum) {
    const float Ah = a.A[h];
    for (int s = threadIdx.x; s < a.S; s += blockDim.x)
        acum[s] = dt_at(a, b, t0 + s, h) * Ah;
    __syncthreads();
    block_inclusive_scan(acum, a.S);
}

template <typename T, int N, int P>
__global__ void __launch_bounds__(kThreads) chunk_state_kernel(ScanArgs a) {
    static_assert(N % 16 == 0 && P % 16 == 0, "N and P must be multiples of 16");
    constexpr int TS = 32;             // tokens per smem tile
    constexpr int RN = N / 16, RP = P / 16;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int S = a.S, C = (a.L + S - 1) / S, t0 = c * S;
    extern __shared__ float sm[];
    float* acum = sm;                  // [S]
    float* w = acum + S;               // [S]
    float* Bs = w + S;                 // [TS][N]
    float* Xs = Bs + TS * N;           // [TS][P]
    load_chunk_cumsum(a, b, h, t0, acum);
    const float aend = acum[S - 1];
    for (int s = threadIdx.x; s < S; s += blockDim.x)
        w[s] = expf(aend - acum[s]) * dt_at(a, b, t0 + s, h);
    __syncthreads();

    const T* x = static_cast<const T*>(a.x);
    const T* Bm = static_cast<const T*>(a.Bm);
    const int tp = threadIdx.x % 16, tn = threadIdx.x / 16;
    float acc[RN][RP];
#pragma unroll
    for (int i = 0; i < RN; ++i)
#pragma unroll
        for (int j = 0; j < RP; ++j) acc[i][j] = 0.f;

    for (int s0 = 0; s0 < S; s0 += TS) {
        for (int e = threadIdx.x; e < TS * N; e += blockDim.x) {
            const int s = e / N, n = e % N;
            const int t = t0 + s0 + s;
            Bs[e] = t < a.L ? ldf(Bm + (((size_t)b * a.L + t) * a.G + group_of(h, a.H, a.G)) * N + n) : 0.f;
        }
        for (int e = threadIdx.x; e < TS * P; e += blockDim.x) {
            const int s = e / P, p = e % P;
            const int t = t0 + s0 + s;
            Xs[e] = t < a.L ? w[s0 + s] * ldf(x + (((size_t)b * a.L + t) * a.H + h) * P + p) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int s = 0; s < TS; ++s) {
            float bv[RN], xv[RP];
#pragma unroll
            for (int i = 0; i < RN; ++i) bv[i] = Bs[s * N + tn + 16 * i];
#pragma unroll
            for (int j = 0; j < RP; ++j) xv[j] = Xs[s * P + tp + 16 * j];
#pragma unroll
            for (int i = 0; i < RN; ++i)
#pragma unroll
                for (int j = 0; j < RP; ++j) acc[i][j] = fmaf(bv[i], xv[j], acc[i][j]);
        }
        __syncthreads();
    }
    const size_t base = (((size_t)b * a.H + h) * C + c) * (size_t)N * P;
    T* dH = static_cast<T*>(a.dH);
#pragma unroll
    for (int i = 0; i < RN; ++i)
#pragma unroll
        for (int j = 0; j < RP; ++j) {
            const size_t idx = base + (size_t)(tn + 16 * i) * P + tp + 16 * j;
            dH[idx] = Elem<T>::from_f(acc[i][j]);
            a.states[idx] = acc[i][j];
        }
    if (threadIdx.x == 0) a.asum[((size_t)b * a.H + h) * C + c] = aend;
}

template <int N, int P>
__global__ void __launch_bounds__(kThreads) state_pass_kernel(ScanArgs a) {
    const int h = blockIdx.y, b = blockIdx.z;
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= N * P) return;
    const int C = (a.L + a.S - 1) / a.S;
    const size_t bh = (size_t)b * a.H + h;
    float prev = a.init_state ? a.init_state[bh * N * P + idx] : 0.f;
    float* st = a.states + bh * (size_t)C * N * P + idx;
    const float* asum = a.asum + bh * C;
    for (int c = 0; c < C; ++c) {
        const float v = fmaf(expf(asum[c]), prev, st[(size_t)c * N * P]);
        st[(size_t)c * N * P] = v;
        prev = v;
    }
}

template <typename T, int N, int P>
__global__ void __launch_bounds__(kThreads) chunk_output_kernel(ScanArgs a) {
    constexpr int TQ = 64;             // query tokens per block
    constexpr int TS = 32;             // source tokens per smem tile
    constexpr int NP = N + 1;          // padded row stride (bank spread)
    constexpr int PT = P / 4;          // outputs per thread (4 threads per token)
    const int S = a.S, C = (a.L + S - 1) / S;
    const int tiles_per_chunk = S / TQ;
    const int c = blockIdx.x / tiles_per_chunk;
    const int q0 = (blockIdx.x % tiles_per_chunk) * TQ;  // first query, chunk-local
    const int h = blockIdx.y, b = blockIdx.z;
    const int t0 = c * S;
    extern __shared__ float sm[];
    float* acum = sm;                  // [S]
    float* Cs = acum + S;              // [TQ][NP]
    float* Bs = Cs + TQ * NP;          // [TS][NP]
    float* Xs = Bs + TS * NP;          // [TS][P]  (dt_s x_s)
    float* Ms = Xs + TS * P;           // [TQ][TS]
    float* Hs = Bs;                    // [N][P], reuses Bs/Xs/Ms after the loop
    const T* x = static_cast<const T*>(a.x);
    const T* Bm = static_cast<const T*>(a.Bm);
    const T* Cm = static_cast<const T*>(a.Cm);

    load_chunk_cumsum(a, b, h, t0, acum);
    for (int e = threadIdx.x; e < TQ * N; e += blockDim.x) {
        const int t = e / N, n = e % N;
        const int tok = t0 + q0 + t;
        Cs[t * NP + n] = tok < a.L ? ldf(Cm + (((size_t)b * a.L + tok) * a.G + group_of(h, a.H, a.G)) * N + n) : 0.f;
    }
    const int tl = threadIdx.x / 4, pg = threadIdx.x % 4;
    const int tq = q0 + tl;            // chunk-local query index
    float acc[PT];
#pragma unroll
    for (int j = 0; j < PT; ++j) acc[j] = 0.f;

    for (int s0 = 0; s0 < q0 + TQ; s0 += TS) {
        __syncthreads();
        for (int e = threadIdx.x; e < TS * N; e += blockDim.x) {
            const int s = e / N, n = e % N;
            const int t = t0 + s0 + s;
            Bs[s * NP + n] = t < a.L ? ldf(Bm + (((size_t)b * a.L + t) * a.G + group_of(h, a.H, a.G)) * N + n) : 0.f;
        }
        for (int e = threadIdx.x; e < TS * P; e += blockDim.x) {
            const int s = e / P, p = e % P;
            const int t = t0 + s0 + s;
            const size_t tok = (size_t)b * a.L + t;
            Xs[e] = t < a.L ? a.dt[tok * a.H + h] * ldf(x + (tok * a.H + h) * P + p) : 0.f;
        }
        __syncthreads();
        // masked, decayed C.B for TQ x TS pairs: 8 per thread
        for (int e = threadIdx.x; e < TQ * TS; e += blockDim.x) {
            const int t = e / TS, s = e % TS;
            float v = 0.f;
            if (s0 + s <= q0 + t) {
                float g = 0.f;
#pragma unroll 8
                for (int n = 0; n < N; ++n) g = fmaf(Cs[t * NP + n], Bs[s * NP + n], g);
                v = g * expf(acum[q0 + t] - acum[s0 + s]);
            }
            Ms[e] = v;
        }
        __syncthreads();
        const int smax = min(TS, tq - s0 + 1);
        for (int s = 0; s < smax; ++s) {
            const float m = Ms[tl * TS + s];
#pragma unroll
            for (int j = 0; j < PT; ++j) acc[j] = fmaf(m, Xs[s * P + pg * PT + j], acc[j]);
        }
    }
    // inter-chunk term from the boundary state before this chunk
    const float* hprev = nullptr;
    if (c > 0) hprev = a.states + (((size_t)b * a.H + h) * C + c - 1) * (size_t)N * P;
    else if (a.init_state) hprev = a.init_state + ((size_t)b * a.H + h) * (size_t)N * P;
    if (hprev) {
        __syncthreads();
        for (int e = threadIdx.x; e < N * P; e += blockDim.x) Hs[e] = hprev[e];
        __syncthreads();
        const float scale = expf(acum[tq]);
        float off[PT];
#pragma unroll
        for (int j = 0; j < PT; ++j) off[j] = 0.f;
        for (int n = 0; n < N; ++n) {
            const float cv = Cs[tl * NP + n];
#pragma unroll
            for (int j = 0; j < PT; ++j) off[j] = fmaf(cv, Hs[n * P + pg * PT + j], off[j]);
        }
#pragma unroll
        for (int j = 0; j < PT; ++j) acc[j] = fmaf(scale, off[j], acc[j]);
    }
    if (t0 + tq >= a.L) return;   // a row past the end of a partial last chunk
    float* y = a.y + (((size_t)b * a.L + t0 + tq) * a.H + h) * P + pg * PT;
#pragma unroll
    for (int j = 0; j < PT; ++j) y[j] = acc[j];
}

template <typename T, int N, int P>
cudaError_t run(const ScanArgs& a, cudaStream_t st) {
    const int C = (a.L + a.S - 1) / a.S;
    {
        const size_t smem = sizeof(float) * (2 * a.S + 32 * N + 32 * P);
        auto k = chunk_state_kernel<T, N, P>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k<<<dim3(C, a.H, a.B), kThreads, smem, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launches(1);
    }
    {
        state_pass_kernel<N, P><<<dim3((N * P + kThreads - 1) / kThreads, a.H, a.B), kThreads, 0, st>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        count_launches(1);
    }
    {
        constexpr int NP = N + 1;
        size_t loop = sizeof(float) * (32 * NP + 32 * P + 64 * 32);
        const size_t hs = sizeof(float) * N * P;
        if (hs > loop) loop = hs;
        const size_t smem = sizeof(float) * (a.S + 64 * NP) + loop;
        auto k = chunk_output_kernel<T, N, P>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k<<<dim3(C * (a.S / 64), a.H, a.B), kThreads, smem, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launches(1);
    }
    return cudaSuccess;
}

}  // namespace

bool ssd_scan_supported(int N, int P, int S, dart_dtype) {
    const bool np = (N == 16 && P == 16) || (N == 64 && P == 64) || (N == 128 && P == 64);
    return np && (S == 64 || S == 128 || S == 256);
}

cudaError_t launch_ssd_scan(const ScanArgs& a, dart_dtype dt, cudaStream_t st) {
    if (ssd_scan_tc_applicable(a.N, a.P, a.S, dt)) return launch_ssd_scan_tc(a, st);
#define DART_SCAN_CASE(NN, PP)                                                      \
    if (a.N == NN && a.P == PP)                                                     \
        return dt == DART_F32 ? run<float, NN, PP>(a, st) : run<__nv_bfloat16, NN, PP>(a, st);
    DART_SCAN_CASE(16, 16)
    DART_SCAN_CASE(64, 64)
    DART_SCAN_CASE(128, 64)
#undef DART_SCAN_CASE
    return cudaErrorInvalidValue;
}

}  // namespace dart
