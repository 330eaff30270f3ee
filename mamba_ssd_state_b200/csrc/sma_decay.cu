// sma_decay.cu -- decay terms for the decayed-memory variant of SMA.
//
// Referee major comment 3 on SMA Eq. (8) (Pith review of DART) contrasts the
// raw chunk memories that SMA reads with memories carried forward to the query
// token by the recurrence's own decay:
//   dH[c]  ->  exp(sum_{r=e(c)+1}^{t} dt_r A_h) dH[c],
// which is the share of dH[c] still present in the state H_t.  For token t of
// chunk k the exponent splits into t's prefix inside chunk k plus the full
// sums of the chunks between c and k:
//   la2[b,h,t]   = log2(e) * sum_{r=kS}^{t} dt_r A_h          fp32, 0 past L
//   gpre[b,h,j]  = sum_{c'<j} la2[b,h,c'S + S-1]               fp64
//   base-2 exponent of memory c at t = la2[b,h,t] + gpre[b,h,k] - gpre[b,h,c+1].
// The chunk-level prefix is fp64 so that subtracting two long prefixes keeps
// full fp32 accuracy in the result; the SMA kernels round it once per memory.
//
// Layouts: dt [B,L,H], A [H]; la2 [B,H,C,S] (C = ceil(L/S)); gpre [B,H,C].
#include "dart_common.cuh"

namespace dart {
namespace {

constexpr int kHeadsPerCta = 8;

// One CTA per (chunk, batch, group of 8 heads): the chunk's dt slice of those
// heads is read once, coalesced along heads, into shared memory; then one warp
// per head scans its S tokens (S/32 consecutive tokens per lane).
__global__ void __launch_bounds__(32 * kHeadsPerCta)
    decay_prefix_kernel(int L, int H, int S, const float* __restrict__ dt, const float* __restrict__ A,
                        float* __restrict__ la2) {
    extern __shared__ float a_s[];   // [S][kHeadsPerCta + 1]
    constexpr int kLd = kHeadsPerCta + 1;
    const int c = blockIdx.x, b = blockIdx.y, h0 = blockIdx.z * kHeadsPerCta;
    const int C = gridDim.x;
    for (int i = threadIdx.x; i < S * kHeadsPerCta; i += blockDim.x) {
        const int s = i / kHeadsPerCta, hh = i % kHeadsPerCta;
        const int t = c * S + s, h = h0 + hh;
        a_s[s * kLd + hh] = (t < L && h < H) ? dt[((size_t)b * L + t) * H + h] * A[h] : 0.f;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = h0 + warp;
    if (h >= H) return;
    const int per = S / 32;               // S is a multiple of 32
    float loc[8];
    float run = 0.f;
    for (int j = 0; j < per; ++j) {
        run += a_s[(lane * per + j) * kLd + warp];
        loc[j] = run;
    }
    // exclusive scan of the lane totals
    float incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    const float base = incl - run;
    float* dst = la2 + (((size_t)b * H + h) * C + c) * S + lane * per;
    for (int j = 0; j < per; ++j) dst[j] = kLog2e * (base + loc[j]);
}

// One warp per (b, h): gpre[j] = sum of the chunk totals of chunks 0..j-1, in
// fp64, 32 chunks per round with the running carry.
__global__ void __launch_bounds__(256)
    decay_chunk_prefix_kernel(int BH, int C, int S, const float* __restrict__ la2, double* __restrict__ gpre) {
    const int bh = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (bh >= BH) return;
    const float* tot = la2 + (size_t)bh * C * S + (S - 1);   // chunk totals at stride S
    double carry = 0.0;
    for (int base = 0; base < C; base += 32) {
        const int j = base + lane;
        double v = (j >= 1 && j < C) ? (double)tot[(size_t)(j - 1) * S] : 0.0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        if (j < C) gpre[(size_t)bh * C + j] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
    }
}

}  // namespace

size_t sma_decay_workspace_bytes(int B, int L, int H, int S) {
    if (B <= 0 || L <= 0 || H <= 0 || S <= 0) return 0;
    const size_t C = (size_t)(L + S - 1) / S;
    const size_t la2 = ((sizeof(float) * (size_t)B * H * C * S) + 255) & ~size_t(255);
    return la2 + sizeof(double) * (size_t)B * H * C;
}

cudaError_t launch_sma_decay_terms(int B, int L, int H, int S, const float* dt, const float* A, float* la2,
                                   double* gpre, cudaStream_t st) {
    if (S % 32 != 0 || S > 256) return cudaErrorInvalidValue;
    const int C = (L + S - 1) / S;
    const size_t smem = sizeof(float) * (size_t)S * (kHeadsPerCta + 1);
    decay_prefix_kernel<<<dim3(C, B, (H + kHeadsPerCta - 1) / kHeadsPerCta), 32 * kHeadsPerCta, smem, st>>>(
        L, H, S, dt, A, la2);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int BH = B * H;
    decay_chunk_prefix_kernel<<<(BH + 7) / 8, 256, 0, st>>>(BH, C, S, la2, gpre);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launches(2);
    return cudaSuccess;
}

}  // namespace dart
