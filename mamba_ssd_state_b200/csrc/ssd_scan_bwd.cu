// ssd_scan_bwd.cu -- gradients through the SSD scan with retained chunk
// memories (the training pass the DART abstract claims), on CUDA cores.
//
// Forward (Mamba-2 SSD recurrence, SSD view Eq. (4) cited by the Pith review
// of DART), per (b, h), a_t = exp(dt_t A_h), u_t = dt_t B_t x_t^T:
//   H_t = a_t H_{t-1} + u_t (H_{-1} = init),  y_t = H_t^T C_t
//   D_t = a_t D_{t-1} + u_t, D restarted at every chunk's first token,
//   dH[c] = D at the chunk's last token e(c).
// Backward of sum(dy * y) + sum(gD * dH) (gD: the memory gradients SMA's
// backward returns), by the adjoint recurrences run from the last token:
//   G_t = C_t dy_t^T + a_{t+1} G_{t+1}               (dLoss/dH_t)
//   K_t = gD[c] at t = e(c), else a_{t+1} K_{t+1}     (dLoss/dD_t, inside chunk c)
//   Z_t = G_t + K_t
//   dx_t = dt_t Z_t^T B_t      dB_t = sum_h dt_t Z_t x_t      dC_t = sum_h H_t dy_t
//   ddt_t = sum(Z_t o B_t x_t^T) + A_h a_t (sum(G_t o H_{t-1}) + sum(K_t o D_{t-1}))
//   dA_h  = sum_{b,t} dt_t a_t (sum(G_t o H_{t-1}) + sum(K_t o D_{t-1}))
//   dinit = a_0 G_0
// (D_{t-1} = 0 at a chunk's first token.)
//
// ssd_scan_bwd_kernel: one CTA per (b, h), each thread one state row n and 8
// consecutive value columns.  Chunks are taken last to first: the chunk's
// H_{t-1} and D_{t-1} are recomputed forward from the boundary state the
// forward stored (states[c-1], or init / zero) into a scratch history, then
// the adjoints walk the chunk backwards.  Per token, dx (a sum over rows) and
// the ddt terms (sums over the whole state) are reduced with warp shuffles and
// one shared-memory exchange; dB and dC (sums over columns) with shuffles
// among the lanes of a row, written per head and summed over heads after.
#include "dart_backward.cuh"

namespace dart {
namespace {

constexpr int kCols = 8;     // value columns per thread
constexpr int kTT = 32;      // tokens per shared-memory tile

template <typename T, int N, int P>
__global__ void __launch_bounds__(N * P / kCols) ssd_scan_bwd_kernel(ScanBwdArgs a) {
    constexpr int CG = P / kCols;              // threads per state row
    constexpr int NT = N * P / kCols;          // threads
    constexpr int NW = NT / 32;                // warps
    static_assert(P % kCols == 0 && 32 % CG == 0 && NT % 32 == 0, "unsupported (N, P)");
    const int L = a.L, H = a.H, S = a.S, C = (L + S - 1) / S;
    const int h = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = tid / CG, p0 = (tid % CG) * kCols;
    const size_t bh = (size_t)b * H + h;
    extern __shared__ __align__(16) float sm[];
    float* Bs = sm;                            // [kTT][N]
    float* Cs = Bs + kTT * N;                  // [kTT][N]
    float* xs = Cs + kTT * N;                  // [kTT][P]
    float* ys = xs + kTT * P;                  // [kTT][P]  dy
    float* dts = ys + kTT * P;                 // [kTT]
    float* red = dts + kTT;                    // [2][NW][P + 2]
    const T* x = static_cast<const T*>(a.x);
    const T* Bm = static_cast<const T*>(a.Bm);
    const T* Cm = static_cast<const T*>(a.Cm);
    const float Ah = a.A[h];
    float* histH = a.hist + bh * (size_t)S * N * P;
    float* histD = histH + (size_t)a.B * H * S * N * P;

    auto stage = [&](int tb) {   // tokens tb .. tb + kTT - 1 (zeros past L)
        __syncthreads();
        for (int i = tid; i < kTT * N; i += NT) {
            const int r = i / N, nn = i % N;
            const bool in = tb + r < L;
            const size_t tok = (size_t)b * L + tb + r;
            const size_t tg = tok * a.G + group_of(h, H, a.G);   // B and C of this head's group
            Bs[i] = in ? ldf(Bm + tg * N + nn) : 0.f;
            Cs[i] = in ? ldf(Cm + tg * N + nn) : 0.f;
        }
        for (int i = tid; i < kTT * P; i += NT) {
            const int r = i / P, pp = i % P;
            const bool in = tb + r < L;
            const size_t tok = (size_t)b * L + tb + r;
            xs[i] = in ? ldf(x + (tok * H + h) * P + pp) : 0.f;
            ys[i] = in ? a.dy[(tok * H + h) * P + pp] : 0.f;
        }
        for (int r = tid; r < kTT; r += NT) dts[r] = tb + r < L ? a.dt[((size_t)b * L + tb + r) * H + h] : 0.f;
        __syncthreads();
    };

    float G[kCols], K[kCols];                  // a_{t+1} G_{t+1} and a_{t+1} K_{t+1} carried down
#pragma unroll
    for (int j = 0; j < kCols; ++j) G[j] = K[j] = 0.f;
    float dA_acc = 0.f;
    int rb = 0;                                // reduction buffer parity
    for (int c = C - 1; c >= 0; --c) {
        const int s0 = c * S, e = min(L, s0 + S) - 1;
        // ---- forward recompute of H_{t-1}, D_{t-1} over the chunk ----------
        float Hc[kCols], Dc[kCols];
        {
            const float* src = c > 0 ? a.states + ((bh * C + (c - 1)) * N + n) * (size_t)P + p0
                                     : (a.init ? a.init + (bh * N + n) * (size_t)P + p0 : nullptr);
#pragma unroll
            for (int j = 0; j < kCols; ++j) {
                Hc[j] = src ? src[j] : 0.f;
                Dc[j] = 0.f;
            }
        }
        for (int tb = s0; tb <= e; tb += kTT) {
            stage(tb);
            for (int r = 0; r < kTT && tb + r <= e; ++r) {
                float* hH = histH + (size_t)(tb + r - s0) * N * P + (size_t)n * P + p0;
                float* hD = histD + (size_t)(tb + r - s0) * N * P + (size_t)n * P + p0;
#pragma unroll
                for (int j = 0; j < kCols; ++j) {
                    hH[j] = Hc[j];
                    hD[j] = Dc[j];
                }
                const float dtt = dts[r], at = expf(dtt * Ah), bn = dtt * Bs[r * N + n];
#pragma unroll
                for (int j = 0; j < kCols; ++j) {
                    const float u = bn * xs[r * P + p0 + j];
                    Hc[j] = fmaf(at, Hc[j], u);
                    Dc[j] = fmaf(at, Dc[j], u);
                }
            }
        }
        // ---- adjoints, last token of the chunk to the first ---------------
        const float* gD = a.ddH ? a.ddH + ((bh * C + c) * N + n) * (size_t)P + p0 : nullptr;
#pragma unroll
        for (int j = 0; j < kCols; ++j) K[j] = gD ? gD[j] : 0.f;   // K_e = gD[c]
        const int ntile = (e - s0) / kTT;
        for (int ti = ntile; ti >= 0; --ti) {
            const int tb = s0 + ti * kTT;
            stage(tb);
            for (int r = min(kTT - 1, e - tb); r >= 0; --r) {
                const int t = tb + r;
                const float* hH = histH + (size_t)(t - s0) * N * P + (size_t)n * P + p0;
                const float* hD = histD + (size_t)(t - s0) * N * P + (size_t)n * P + p0;
                const float dtt = dts[r], at = expf(dtt * Ah);
                const float bnr = Bs[r * N + n], cn = Cs[r * N + n];
                float dxp[kCols], zx = 0.f, hdy = 0.f, q2 = 0.f;
#pragma unroll
                for (int j = 0; j < kCols; ++j) {
                    const float xv = xs[r * P + p0 + j], dyv = ys[r * P + p0 + j];
                    const float hprev = hH[j], dprev = hD[j];
                    const float Gt = fmaf(cn, dyv, G[j]);
                    const float Zt = Gt + K[j];
                    dxp[j] = bnr * Zt;
                    zx = fmaf(Zt, xv, zx);
                    hdy = fmaf(fmaf(at, hprev, dtt * bnr * xv), dyv, hdy);   // H_t . dy
                    q2 = fmaf(Gt, hprev, fmaf(K[j], dprev, q2));
                    G[j] = at * Gt;                                           // for token t - 1
                    K[j] = t == s0 ? 0.f : at * K[j];
                }
                // dB, dC for this head: sum over the CG lanes of row n
#pragma unroll
                for (int o = 1; o < CG; o <<= 1) {
                    zx += __shfl_xor_sync(0xffffffffu, zx, o);
                    hdy += __shfl_xor_sync(0xffffffffu, hdy, o);
                }
                if (tid % CG == 0) {
                    const size_t o = (((size_t)b * L + t) * H + h) * N + n;
                    a.dBh[o] = dtt * zx;
                    a.dCh[o] = hdy;
                }
                // dx: sum over rows of the lanes with the same columns; ddt terms: whole warp
                float q1 = bnr * zx;   // this row's sum(Z o B x^T), counted once per row below
                if (tid % CG != 0) q1 = 0.f;
#pragma unroll
                for (int o = CG; o < 32; o <<= 1)
#pragma unroll
                    for (int j = 0; j < kCols; ++j) dxp[j] += __shfl_xor_sync(0xffffffffu, dxp[j], o);
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    q1 += __shfl_xor_sync(0xffffffffu, q1, o);
                    q2 += __shfl_xor_sync(0xffffffffu, q2, o);
                }
                float* rw = red + (size_t)rb * NW * (P + 2) + (size_t)warp * (P + 2);
                if (lane < CG) {
#pragma unroll
                    for (int j = 0; j < kCols; ++j) rw[p0 + j] = dxp[j];
                }
                if (lane == 0) {
                    rw[P] = q1;
                    rw[P + 1] = q2;
                }
                __syncthreads();
                const float* rr = red + (size_t)rb * NW * (P + 2);
                const size_t tok = (size_t)b * L + t;
                if (tid < P) {
                    float sdx = 0.f;
                    for (int w = 0; w < NW; ++w) sdx += rr[w * (P + 2) + tid];
                    a.dx[(tok * H + h) * P + tid] = dtt * sdx;
                }
                if (tid == 0) {
                    float s1 = 0.f, s2 = 0.f;
                    for (int w = 0; w < NW; ++w) {
                        s1 += rr[w * (P + 2) + P];
                        s2 += rr[w * (P + 2) + P + 1];
                    }
                    a.ddt[tok * H + h] = s1 + Ah * at * s2;
                    dA_acc = fmaf(dtt * at, s2, dA_acc);
                }
                rb ^= 1;   // the other buffer next token: one barrier per token suffices
            }
        }
    }
    // dLoss/dH_{-1} = a_0 G_0, which is what G carries now
    if (a.dinit) {
        float* dst = a.dinit + (bh * N + n) * (size_t)P + p0;
#pragma unroll
        for (int j = 0; j < kCols; ++j) dst[j] = G[j];
    }
    if (tid == 0) a.dApart[bh] = dA_acc;
}

// dB, dC [B,L,G,N] summed over the heads of each group (dC plus dC_add when
// given); dA summed over the batch (fixed order).
__global__ void scan_bwd_reduce(ScanBwdArgs a, int N) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t nbc = (size_t)a.B * a.L * a.G * N;
    if (i < nbc) {
        const size_t tok = i / ((size_t)a.G * N), nn = i % N;
        const int g = (int)((i / N) % a.G), hg = a.H / a.G;
        float sb = 0.f, sc = 0.f;
        for (int h = g * hg; h < (g + 1) * hg; ++h) {
            sb += a.dBh[(tok * a.H + h) * N + nn];
            sc += a.dCh[(tok * a.H + h) * N + nn];
        }
        if (a.dC_add) sc += a.dC_add[i];   // read before the write: dC_add may be dC itself
        a.dB[i] = sb;
        a.dC[i] = sc;
    }
    if (i < (size_t)a.H) {
        float s = 0.f;
        for (int bb = 0; bb < a.B; ++bb) s += a.dApart[(size_t)bb * a.H + i];
        a.dA[i] = s;
    }
}

template <typename T, int N, int P>
cudaError_t run(const ScanBwdArgs& a, cudaStream_t st) {
    constexpr int NT = N * P / kCols;
    const size_t smem = sizeof(float) * (kTT * (2 * N + 2 * P) + kTT + 2 * (NT / 32) * (P + 2));
    auto k = ssd_scan_bwd_kernel<T, N, P>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<dim3(a.H, a.B), NT, smem, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t n = (size_t)a.B * a.L * a.G * N;
    const size_t m = n > (size_t)a.H ? n : (size_t)a.H;
    scan_bwd_reduce<<<(unsigned)((m + 255) / 256), 256, 0, st>>>(a, N);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launches(2);
    return cudaSuccess;
}

}  // namespace

size_t scan_bwd_workspace_bytes(int B, int L, int H, int N, int P, int S) {
    if (B <= 0 || L <= 0 || H <= 0 || N <= 0 || P <= 0 || S <= 0) return 0;
    auto pad = [](size_t bytes) { return (bytes + 255) & ~size_t(255); };
    return 2 * pad(sizeof(float) * B * H * S * N * P)     // H_{t-1}, D_{t-1} of one chunk per (b, h)
           + 2 * pad(sizeof(float) * B * L * H * N)       // dB, dC per head
           + pad(sizeof(float) * B * H);                  // dA per (b, h)
}

bool scan_bwd_supported(int N, int P) { return (N == 128 && P == 64) || (N == 64 && P == 64) || (N == 16 && P == 16); }

cudaError_t launch_ssd_scan_bwd(ScanBwdArgs a, void* workspace, dart_dtype dt, cudaStream_t st) {
    auto pad = [](size_t bytes) { return (bytes + 255) & ~size_t(255); };
    uint8_t* w = static_cast<uint8_t*>(workspace);
    a.hist = reinterpret_cast<float*>(w);                 // H history, then D history right after it
    w += 2 * pad(sizeof(float) * a.B * a.H * a.S * a.N * a.P);
    a.dBh = reinterpret_cast<float*>(w);
    w += pad(sizeof(float) * a.B * a.L * a.H * a.N);
    a.dCh = reinterpret_cast<float*>(w);
    w += pad(sizeof(float) * a.B * a.L * a.H * a.N);
    a.dApart = reinterpret_cast<float*>(w);
#define DART_SCAN_BWD_CASE(NN, PP)                                                  \
    if (a.N == NN && a.P == PP)                                                     \
        return dt == DART_F32 ? run<float, NN, PP>(a, st) : run<__nv_bfloat16, NN, PP>(a, st);
    DART_SCAN_BWD_CASE(16, 16)
    DART_SCAN_BWD_CASE(64, 64)
    DART_SCAN_BWD_CASE(128, 64)
#undef DART_SCAN_BWD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace dart
