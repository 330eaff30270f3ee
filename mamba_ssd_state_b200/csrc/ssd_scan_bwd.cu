// ssd_scan_bwd.cu -- gradients through the SSD scan with retained chunk
// memories (the training pass the DART abstract claims), chunk-parallel on
// CUDA cores.
//
// Forward (Mamba-2 SSD recurrence, SSD view Eq. (4) cited by the Pith review
// of DART), per (b, h), l_t = dt_t A_h, a_t = exp(l_t), u_t = dt_t B_t x_t^T:
//   H_t = a_t H_{t-1} + u_t (H_{-1} = init),  y_t = H_t^T C_t
//   D_t = a_t D_{t-1} + u_t, D restarted at every chunk's first token,
//   dH[c] = D at the chunk's last token e(c).
// Backward of sum(dy * y) + sum(gD * dH) (gD: the memory gradients SMA's
// backward returns).  The token-wise adjoints are
//   G_t = C_t dy_t^T + a_{t+1} G_{t+1}   (dLoss/dH_t),   K_t = dLoss/dD_t,
//   dx_t = dt_t (G_t + K_t)^T B_t,  dB_t = sum_h dt_t (G_t + K_t) x_t,
//   dC_t = sum_h H_t dy_t,  dl_t = a_t (sum(G_t o H_{t-1}) + sum(K_t o D_{t-1})),
//   ddt_t = x_t . ((G_t + K_t)^T B_t) + A_h dl_t,  dA_h = sum_{b,t} dt_t dl_t.
// Inside chunk c (tokens s0..e, Acum_t = sum_{r=s0}^{t} l_r, Ae = Acum_e,
// h_in the state entering the chunk) they split into a chunk-local part and
// two matrices known before the chunk is walked:
//   G_t = Gl_t + exp(Ae - Acum_t) Gin[c],  K_t = exp(Ae - Acum_t) gD[c],
//   Gl_t = sum_{s=t}^{e} exp(Acum_s - Acum_t) C_s dy_s^T,
//   Gin[c] = a_{e+1} G_{e+1}: Gin[C-1] = 0, Gin[c-1] = exp(Ae(c)) Gin[c] + dS[c],
//   dS[c] = sum_s exp(Acum_s) C_s dy_s^T,  dinit = Gin[-1];
// and, with R = Gin[c] + gD[c] and H_{t-1} = exp(Acum_{t-1}) h_in + D_{t-1},
//   dl_t = exp(Acum_t) sum(Gl_t o h_in) + Rect_t
//          + exp(Ae - Acum_{t-1}) (exp(Acum_{t-1}) sum(Gin o h_in) + sum(R o D_{t-1})),
//   Rect_t = sum_{r < t <= s} W_{s,r},
//   W_{s,r} = exp(Acum_s - Acum_r) dt_r (C_s . B_r)(dy_s . x_r)   (r < s, same chunk)
// (a_t sum(Gl_t o D_{t-1}) expanded over the tokens of both factors).  So no
// per-token state history is kept:
//   scan_bwd_chunk_adjoint  per (b, h, c): dS[c] by a walk from the chunk's
//                           last token, and Ae(c).
//   scan_bwd_gin_pass       per (b, h, state element): Gin in place of dS,
//                           last chunk to first, and dinit.
//   scan_bwd_rect           per (b, h, c): W in 64 x 64 tiles from C B^T and
//                           dy x^T, its row and column sums, and Rect_t by the
//                           recursion Rect_t = Rect_{t+1} - sum_{s>t} W_{s,t}
//                           + sum_{r<t} W_{t,r}.
//   scan_bwd_walk           per (b, h, c): a forward walk (D_t from zero; dC_t
//                           and the sum(R o D_{t-1}) term per token) and a
//                           backward walk (Gl_t from zero; dx_t, dB_t and the
//                           rest of ddt_t, dA).  Each thread holds one state
//                           row n and 8 consecutive value columns.
//   scan_bwd_reduce         dB, dC summed over the heads of each group, dA
//                           over (b, c), in a fixed order.
#include <type_traits>

#include "dart_backward.cuh"

namespace dart {
namespace {

constexpr int kCols = 8;     // value columns per thread in the walks
constexpr int kTT = 32;      // tokens per shared-memory tile in the walks

// Chunk bounds of (b, c): tokens s0 .. e (e < L).
struct ChunkSpan {
    int s0, e, n;            // n = e - s0 + 1
    __device__ ChunkSpan(int c, int S, int L) : s0(c * S), e(min(L, c * S + S) - 1), n(e - s0 + 1) {}
};

// Inclusive prefix of l_t = dt_t A_h over the chunk into acum[0..S) (slots
// past the chunk's end repeat the last value); warp 0 only.
__device__ void chunk_acum(const ScanBwdArgs& a, int b, int h, const ChunkSpan& cs, float* acum) {
    const int lane = threadIdx.x & 31;
    const float Ah = a.A[h];
    const int per = (a.S + 31) / 32, t0 = lane * per;
    float run = 0.f;
    for (int i = 0; i < per && t0 + i < a.S; ++i) {
        const int t = t0 + i;
        run += t < cs.n ? a.dt[((size_t)b * a.L + cs.s0 + t) * a.H + h] * Ah : 0.f;
        acum[t] = run;
    }
    float off = run;   // exclusive prefix of the lane totals
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float v = __shfl_up_sync(0xffffffffu, off, o);
        if (lane >= o) off += v;
    }
    off -= run;
    for (int i = 0; i < per && t0 + i < a.S; ++i) acum[t0 + i] += off;
}

// Stages tokens tb .. tb + kTT - 1 of (b, h) into shared memory (zeros past
// the chunk's end): B, C rows of the head's group, x, dy rows, dt.
template <typename T, int N, int P>
struct Stage {
    float *Bs, *Cs, *xs, *ys, *dts;
    __device__ void operator()(const ScanBwdArgs& a, int b, int h, int tb, int tend, int NT, bool wantB, bool wantC,
                               bool wantX) {
        const int tid = threadIdx.x;
        const T* x = static_cast<const T*>(a.x);
        const T* Bm = static_cast<const T*>(a.Bm);
        const T* Cm = static_cast<const T*>(a.Cm);
        const int grp = group_of(h, a.H, a.G);
        __syncthreads();
        for (int i = tid; i < kTT * N; i += NT) {
            const int r = i / N, nn = i % N;
            const bool in = tb + r <= tend;
            const size_t tg = ((size_t)b * a.L + tb + r) * a.G + grp;
            if (wantB) Bs[i] = in ? ldf(Bm + tg * N + nn) : 0.f;
            if (wantC) Cs[i] = in ? ldf(Cm + tg * N + nn) : 0.f;
        }
        for (int i = tid; i < kTT * P; i += NT) {
            const int r = i / P, pp = i % P;
            const bool in = tb + r <= tend;
            const size_t tok = (size_t)b * a.L + tb + r;
            if (wantX) xs[i] = in ? ldf(x + (tok * a.H + h) * P + pp) : 0.f;
            ys[i] = in ? a.dy[(tok * a.H + h) * P + pp] : 0.f;
        }
        for (int r = tid; r < kTT; r += NT) dts[r] = tb + r <= tend ? a.dt[((size_t)b * a.L + tb + r) * a.H + h] : 0.f;
        __syncthreads();
    }
};

// ---------------------------------------------------------------------------
// dS[c] = sum_s exp(Acum_s) C_s dy_s^T, walked from the chunk's last token
// (carry = a_t (C_t dy_t^T + carry)), and Ae(c).
// ---------------------------------------------------------------------------
template <typename T, int N, int P>
__global__ void __launch_bounds__(N * P / kCols) scan_bwd_chunk_adjoint(ScanBwdArgs a) {
    constexpr int CG = P / kCols, NT = N * P / kCols;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, C = gridDim.x;
    const int tid = threadIdx.x, n = tid / CG, p0 = (tid % CG) * kCols;
    const size_t bhc = ((size_t)b * a.H + h) * C + c;
    const ChunkSpan cs(c, a.S, a.L);
    extern __shared__ __align__(16) float sm[];
    Stage<T, N, P> st{nullptr, sm, nullptr, sm + kTT * N, sm + kTT * N + kTT * P};
    if (tid < 32) {   // Ae = sum of l over the chunk
        float s = 0.f;
        for (int t = tid; t < cs.n; t += 32) s += a.dt[((size_t)b * a.L + cs.s0 + t) * a.H + h];
        s = warp_sum(s);
        if (tid == 0) a.asum[bhc] = s * a.A[h];
    }
    const float Ah = a.A[h];
    float carry[kCols];
#pragma unroll
    for (int j = 0; j < kCols; ++j) carry[j] = 0.f;
    for (int ti = (cs.n - 1) / kTT; ti >= 0; --ti) {
        const int tb = cs.s0 + ti * kTT;
        st(a, b, h, tb, cs.e, NT, false, true, false);
        for (int r = min(kTT - 1, cs.e - tb); r >= 0; --r) {
            const float at = expf(st.dts[r] * Ah), cn = st.Cs[r * N + n];
#pragma unroll
            for (int j = 0; j < kCols; ++j) carry[j] = at * fmaf(cn, st.ys[r * P + p0 + j], carry[j]);
        }
    }
    float* dst = a.gin + (bhc * N + n) * (size_t)P + p0;
#pragma unroll
    for (int j = 0; j < kCols; ++j) dst[j] = carry[j];
}

// ---------------------------------------------------------------------------
// Gin[c] in place of dS[c], last chunk to first; dinit = Gin[-1].
// ---------------------------------------------------------------------------
// Eight chunks' dS are loaded before any of them is used, so the loads of a
// group are in flight together instead of one after another.
__global__ void scan_bwd_gin_pass(ScanBwdArgs a, int C) {
    constexpr int kG = 8;
    const size_t NP = (size_t)a.N * a.P;
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (size_t)a.B * a.H * NP) return;
    const size_t bh = i / NP, e = i % NP;
    float* __restrict__ gin = a.gin + bh * C * NP + e;
    const float* __restrict__ asum = a.asum + bh * C;
    float g = 0.f;
    for (int top = C - 1; top >= 0; top -= kG) {
        float ds[kG], dec[kG];
#pragma unroll
        for (int j = 0; j < kG; ++j) {
            const int c = top - j;
            ds[j] = c >= 0 ? gin[(size_t)c * NP] : 0.f;
            dec[j] = c >= 0 ? expf(asum[c]) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < kG; ++j) {
            const int c = top - j;
            if (c < 0) break;
            gin[(size_t)c * NP] = g;
            g = fmaf(dec[j], g, ds[j]);
        }
    }
    if (a.dinit) a.dinit[bh * NP + e] = g;
}

// ---------------------------------------------------------------------------
// Rect_t of every token of (b, h, c) from W_{s,r} = exp(Acum_s - Acum_r) dt_r
// (C_s . B_r)(dy_s . x_r), r < s, in 64 x 64 tiles; 256 threads, each a 4 x 4
// block of (s, r) with rows ty + 16 i and columns tx + 16 j.
// ---------------------------------------------------------------------------
constexpr int kRT = 64;
template <int N, int P>
struct RectSmem {
    static constexpr int KN = N + 4, KP = P + 4;    // padded rows (16-byte aligned)
    static constexpr size_t floats = 4 * 256 /* acum, dt, row, col sums */ + 2 * kRT * KN + 2 * kRT * KP +
                                     16 * kRT /* column partials per ty */;
};

template <typename T, int N, int P>
__global__ void __launch_bounds__(256) scan_bwd_rect(ScanBwdArgs a) {
    using SM = RectSmem<N, P>;
    constexpr int KN = SM::KN, KP = SM::KP;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, C = gridDim.x;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int S = a.S;
    const ChunkSpan cs(c, S, a.L);
    extern __shared__ __align__(16) float sm[];
    float* acum = sm;              // [256]
    float* dtv = acum + 256;       // [256]
    float* rows = dtv + 256;       // [256] sum_{r<s} W_{s,r}
    float* cols = rows + 256;      // [256] sum_{s>r} W_{s,r}
    float* Cs = cols + 256;        // [kRT][KN] C rows of the s tile
    float* Ys = Cs + kRT * KN;     // [kRT][KP] dy rows of the s tile
    float* Bs = Ys + kRT * KP;     // [kRT][KN] B rows of the r tile
    float* Xs = Bs + kRT * KN;     // [kRT][KP] x rows of the r tile
    float* cpart = Xs + kRT * KP;  // [16][kRT] column partials of the 16 ty rows
    const T* x = static_cast<const T*>(a.x);
    const T* Bm = static_cast<const T*>(a.Bm);
    const T* Cm = static_cast<const T*>(a.Cm);
    const int grp = group_of(h, a.H, a.G);
    if (tid < 32) chunk_acum(a, b, h, cs, acum);
    for (int t = tid; t < 256; t += 256) {
        dtv[t] = t < cs.n ? a.dt[((size_t)b * a.L + cs.s0 + t) * a.H + h] : 0.f;
        rows[t] = 0.f;
        cols[t] = 0.f;
    }
    auto load_rows = [&](float* dstN, float* dstP, const T* M, const T* V, bool isDy, int t0) {
        for (int i = tid; i < kRT * N; i += 256) {
            const int r = i / N, k = i % N;
            const bool in = t0 + r < cs.n;
            dstN[r * KN + k] = in ? ldf(M + (((size_t)b * a.L + cs.s0 + t0 + r) * a.G + grp) * N + k) : 0.f;
        }
        for (int i = tid; i < kRT * P; i += 256) {
            const int r = i / P, k = i % P;
            const bool in = t0 + r < cs.n;
            const size_t o = (((size_t)b * a.L + cs.s0 + t0 + r) * a.H + h) * P + k;
            dstP[r * KP + k] = in ? (isDy ? a.dy[o] : ldf(V + o)) : 0.f;
        }
    };
    const int ntile = (cs.n + kRT - 1) / kRT;
    for (int si = 0; si < ntile; ++si) {
        __syncthreads();
        load_rows(Cs, Ys, Cm, x, true, si * kRT);
        for (int ri = 0; ri <= si; ++ri) {
            __syncthreads();
            load_rows(Bs, Xs, Bm, x, false, ri * kRT);
            __syncthreads();
            float cb[4][4], yx[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) cb[i][j] = yx[i][j] = 0.f;
#pragma unroll 2
            for (int k = 0; k < N; k += 4) {
                float4 cv[4], bv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) cv[i] = *reinterpret_cast<const float4*>(Cs + (ty + 16 * i) * KN + k);
#pragma unroll
                for (int j = 0; j < 4; ++j) bv[j] = *reinterpret_cast<const float4*>(Bs + (tx + 16 * j) * KN + k);
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        cb[i][j] = fmaf(cv[i].x, bv[j].x, fmaf(cv[i].y, bv[j].y,
                                   fmaf(cv[i].z, bv[j].z, fmaf(cv[i].w, bv[j].w, cb[i][j]))));
            }
#pragma unroll 2
            for (int k = 0; k < P; k += 4) {
                float4 yv[4], xv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) yv[i] = *reinterpret_cast<const float4*>(Ys + (ty + 16 * i) * KP + k);
#pragma unroll
                for (int j = 0; j < 4; ++j) xv[j] = *reinterpret_cast<const float4*>(Xs + (tx + 16 * j) * KP + k);
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        yx[i][j] = fmaf(yv[i].x, xv[j].x, fmaf(yv[i].y, xv[j].y,
                                   fmaf(yv[i].z, xv[j].z, fmaf(yv[i].w, xv[j].w, yx[i][j]))));
            }
            float rsum[4] = {0.f, 0.f, 0.f, 0.f}, csum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int s = si * kRT + ty + 16 * i;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int r = ri * kRT + tx + 16 * j;
                    const float w = r < s && s < cs.n ? expf(acum[s] - acum[r]) * dtv[r] * cb[i][j] * yx[i][j] : 0.f;
                    rsum[i] += w;
                    csum[j] += w;
                }
            }
            // rows: the 16 tx lanes of a half-warp share the rows -> shuffle
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
                for (int o = 1; o < 16; o <<= 1) rsum[i] += __shfl_xor_sync(0xffffffffu, rsum[i], o);
            }
            if (tx == 0) {
#pragma unroll
                for (int i = 0; i < 4; ++i) rows[si * kRT + ty + 16 * i] += rsum[i];   // one writer per row
            }
            // columns: the 16 ty rows of threads -> shared partials, summed in order
#pragma unroll
            for (int j = 0; j < 4; ++j) cpart[ty * kRT + tx + 16 * j] = csum[j];
            __syncthreads();
            if (tid < kRT) {
                float s = 0.f;
                for (int y = 0; y < 16; ++y) s += cpart[y * kRT + tid];
                cols[ri * kRT + tid] += s;
            }
        }
    }
    __syncthreads();
    if (tid == 0) {
        float* rect = a.rect + (((size_t)b * a.H + h) * C + c) * S;
        float R = 0.f;
        for (int t = cs.n - 1; t >= 0; --t) {
            R += rows[t] - cols[t];
            rect[t] = R;
        }
    }
}

// ---------------------------------------------------------------------------
// The two walks of (b, h, c).
// ---------------------------------------------------------------------------
template <typename T, int N, int P>
__global__ void __launch_bounds__(N * P / kCols) scan_bwd_walk(ScanBwdArgs a) {
    constexpr int CG = P / kCols;              // threads per state row
    constexpr int NT = N * P / kCols;          // threads
    constexpr int NW = NT / 32;                // warps
    static_assert(P % kCols == 0 && 32 % CG == 0 && NT % 32 == 0, "unsupported (N, P)");
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, C = gridDim.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = tid / CG, p0 = (tid % CG) * kCols;
    const int S = a.S, H = a.H;
    const size_t bh = (size_t)b * H + h, bhc = bh * C + c;
    const ChunkSpan cs(c, S, a.L);
    extern __shared__ __align__(16) float sm[];
    Stage<T, N, P> st;
    st.Bs = sm;                                // [kTT][N]
    st.Cs = st.Bs + kTT * N;                   // [kTT][N]
    st.xs = st.Cs + kTT * N;                   // [kTT][P]
    st.ys = st.xs + kTT * P;                   // [kTT][P]
    st.dts = st.ys + kTT * P;                  // [kTT]
    float* red = st.dts + kTT;                 // [2][NW][P + 2]
    float* acum = red + 2 * NW * (P + 2);      // [S]
    float* fterm = acum + S;                   // [S]
    float* fw = fterm + S;                     // [S][NW]  per-warp partials of sum(R o D_{t-1})
    float* c0w = fw + (size_t)S * NW;          // [NW]
    const float Ah = a.A[h];

    float R[kCols], hin[kCols];
    {
        const float* gi = a.gin + (bhc * N + n) * (size_t)P + p0;
        const float* gd = a.ddH ? a.ddH + (bhc * N + n) * (size_t)P + p0 : nullptr;
        const float* hi = c > 0 ? a.states + ((bh * C + (c - 1)) * N + n) * (size_t)P + p0
                                : (a.init ? a.init + (bh * N + n) * (size_t)P + p0 : nullptr);
        float c0 = 0.f;
#pragma unroll
        for (int j = 0; j < kCols; ++j) {
            const float g = gi[j];
            hin[j] = hi ? hi[j] : 0.f;
            R[j] = g + (gd ? gd[j] : 0.f);
            c0 = fmaf(g, hin[j], c0);
        }
        c0 = warp_sum(c0);
        if (lane == 0) c0w[warp] = c0;
    }
    if (warp == 0) chunk_acum(a, b, h, cs, acum);
    __syncthreads();
    const float Ae = acum[cs.n - 1];

    // ---- forward walk: D_t from zero; dC_t and sum(R o D_{t-1}) -----------
    {
        float D[kCols];
#pragma unroll
        for (int j = 0; j < kCols; ++j) D[j] = 0.f;
        for (int tb = cs.s0; tb <= cs.e; tb += kTT) {
            st(a, b, h, tb, cs.e, NT, true, false, true);
            for (int r = 0; r < kTT && tb + r <= cs.e; ++r) {
                const int t = tb + r - cs.s0;
                const float dtt = st.dts[r], at = expf(dtt * Ah), bn = dtt * st.Bs[r * N + n];
                const float eh = expf(acum[t]);
                float rd = 0.f, hdy = 0.f;
#pragma unroll
                for (int j = 0; j < kCols; ++j) {
                    rd = fmaf(R[j], D[j], rd);
                    D[j] = fmaf(at, D[j], bn * st.xs[r * P + p0 + j]);
                    hdy = fmaf(fmaf(eh, hin[j], D[j]), st.ys[r * P + p0 + j], hdy);
                }
#pragma unroll
                for (int o = 1; o < CG; o <<= 1) hdy += __shfl_xor_sync(0xffffffffu, hdy, o);
                if (tid % CG == 0) a.dCh[(((size_t)b * a.L + tb + r) * H + h) * N + n] = hdy;
                rd = warp_sum(rd);
                if (lane == 0) fw[(size_t)t * NW + warp] = rd;
            }
        }
    }
    __syncthreads();
    {
        float c0 = 0.f;
        for (int w = 0; w < NW; ++w) c0 += c0w[w];
        for (int t = tid; t < cs.n; t += NT) {
            float s = 0.f;
            for (int w = 0; w < NW; ++w) s += fw[(size_t)t * NW + w];
            const float am1 = t > 0 ? acum[t - 1] : 0.f;
            // exp(Ae - Acum_{t-1}) (exp(Acum_{t-1}) sum(Gin o h_in) + sum(R o D_{t-1}))
            fterm[t] = expf(Ae) * c0 + expf(Ae - am1) * s;
        }
    }

    // ---- backward walk: Gl_t from zero; dx_t, dB_t, ddt_t, dA -----------
    const float* rect = a.rect + bhc * S;
    float carry[kCols];
#pragma unroll
    for (int j = 0; j < kCols; ++j) carry[j] = 0.f;
    float dA_acc = 0.f;
    int rb = 0;
    for (int ti = (cs.n - 1) / kTT; ti >= 0; --ti) {
        const int tb = cs.s0 + ti * kTT;
        st(a, b, h, tb, cs.e, NT, true, true, true);
        for (int r = min(kTT - 1, cs.e - tb); r >= 0; --r) {
            const int t = tb + r - cs.s0;
            const float dtt = st.dts[r], at = expf(dtt * Ah);
            const float bnr = st.Bs[r * N + n], cn = st.Cs[r * N + n];
            const float f = expf(Ae - acum[t]);
            float dxp[kCols], zx = 0.f, gh = 0.f;
#pragma unroll
            for (int j = 0; j < kCols; ++j) {
                const float gl = fmaf(cn, st.ys[r * P + p0 + j], carry[j]);   // Gl_t
                const float z = fmaf(f, R[j], gl);                             // G_t + K_t
                dxp[j] = bnr * z;
                zx = fmaf(z, st.xs[r * P + p0 + j], zx);
                gh = fmaf(gl, hin[j], gh);
                carry[j] = at * gl;                                            // for token t - 1
            }
#pragma unroll
            for (int o = 1; o < CG; o <<= 1) zx += __shfl_xor_sync(0xffffffffu, zx, o);
            if (tid % CG == 0) a.dBh[(((size_t)b * a.L + tb + r) * H + h) * N + n] = dtt * zx;
            float q1 = tid % CG == 0 ? bnr * zx : 0.f;   // this row's x . (Z^T B), once per row
#pragma unroll
            for (int o = CG; o < 32; o <<= 1)
#pragma unroll
                for (int j = 0; j < kCols; ++j) dxp[j] += __shfl_xor_sync(0xffffffffu, dxp[j], o);
            q1 = warp_sum(q1);
            gh = warp_sum(gh);
            float* rw = red + (size_t)rb * NW * (P + 2) + (size_t)warp * (P + 2);
            if (lane < CG) {
#pragma unroll
                for (int j = 0; j < kCols; ++j) rw[p0 + j] = dxp[j];
            }
            if (lane == 0) {
                rw[P] = q1;
                rw[P + 1] = gh;
            }
            __syncthreads();
            const float* rr = red + (size_t)rb * NW * (P + 2);
            const size_t tok = (size_t)b * a.L + tb + r;
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
                const float dl = expf(acum[t]) * s2 + rect[t] + fterm[t];
                a.ddt[tok * H + h] = s1 + Ah * dl;
                dA_acc = fmaf(dtt, dl, dA_acc);
            }
            rb ^= 1;   // the other buffer next token: one barrier per token suffices
        }
    }
    if (tid == 0) a.dApart[bhc] = dA_acc;
}

// The decay gradient of every token of (b, h, c) from the per-token scalars
// the tensor-core kernel leaves (u, v, q1, colsum and the row blocks' parts of
// rowsum; ssd_scan_bwd_tc.cu):
//   Rect_t = Rect_{t+1} + rowsum_t - colsum_t,   gh_t = v_t + a_{t+1} gh_{t+1},
//   rd_t = E_{t-1},  E_t = a_t E_{t-1} + dt_t u_t,
//   dl_t = exp(Acum_t) gh_t + Rect_t + exp(Ae) c0 + exp(Ae - Acum_{t-1}) rd_t,
//   ddt_t = q1_t + A_h dl_t,  dA += dt_t dl_t,
// with a_t = exp(dt_t A_h) (a_S = 0: nothing follows the chunk's last token).
// One warp per chunk; the lanes stage the chunk's scalars in shared memory and
// lane l then owns tokens 8l .. 8l+7.  Each recursion is linear, so each is a
// warp scan: the prefix of dt A and the suffix of rowsum - colsum are sums;
// gh (backward) and E (forward) compose per-lane affine maps x -> K + M x, so
// every lane learns the value entering its tokens and finishes them itself.
__global__ void __launch_bounds__(32) scan_bwd_scalars(ScanBwdArgs a, int C) {
    constexpr int K = 8;        // tokens per lane; the chunk has at most 256
    constexpr unsigned kAll = 0xffffffffu;
    __shared__ float sdt[256], su[256], sv[256], sq[256], srw[256], scl[256];
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, lane = threadIdx.x;
    const size_t bhc = ((size_t)b * a.H + h) * C + c;
    const ChunkSpan cs(c, a.S, a.L);
    const size_t plane = (size_t)a.B * a.H * C * a.S;
    const float* sc = a.rect + bhc * a.S;
    for (int t = lane; t < cs.n; t += 32) {
        sdt[t] = a.dt[((size_t)b * a.L + cs.s0 + t) * a.H + h];
        su[t] = sc[t];
        sv[t] = sc[plane + t];
        sq[t] = sc[2 * plane + t];
        scl[t] = sc[3 * plane + t];
        // rowsum of t: the parts of the row blocks up to t's own (block 0 covers every t)
        srw[t] = sc[4 * plane + t] + (t >= 128 ? sc[5 * plane + t] : 0.f);
    }
    __syncwarp();
    const float Ah = a.A[h];
    const int t0 = K * lane;
    const int nt = max(0, min(K, cs.n - t0));   // this lane's tokens
    float dtv[K], av[K], acum[K];
    float loc = 0.f;
#pragma unroll
    for (int j = 0; j < K; ++j) {
        dtv[j] = j < nt ? sdt[t0 + j] : 0.f;
        av[j] = expf(dtv[j] * Ah);
        loc += dtv[j] * Ah;
        acum[j] = loc;
    }
    // Acum: inclusive prefix of the lanes' sums, then the exclusive part
    float incl = loc;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const float up = __shfl_up_sync(kAll, incl, d);
        if (lane >= d) incl += up;
    }
    float before = __shfl_up_sync(kAll, incl, 1);   // Acum of the token before this lane's first
    if (lane == 0) before = 0.f;
#pragma unroll
    for (int j = 0; j < K; ++j) acum[j] += before;
    const float Ae = __shfl_sync(kAll, incl, 31);
    const float eAc0 = expf(Ae) * a.c0[bhc];
    // a_{t+1} of each of this lane's tokens: the next lane's first for the last
    const float a_first_next = __shfl_down_sync(kAll, av[0], 1);
    auto a_next = [&](int j) -> float {
        if (t0 + j + 1 >= cs.n) return 0.f;
        return j + 1 < K ? av[j + 1] : a_first_next;
    };
    // gh, backward: this lane's map from gh entering from the right to gh at
    // its first token, composed with the maps of the later lanes
    float M = 1.f, Kc = 0.f;
#pragma unroll
    for (int j = K - 1; j >= 0; --j) {
        if (j < nt) {
            const float an = a_next(j);
            Kc = fmaf(an, Kc, sv[t0 + j]);
            M *= an;
        }
    }
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const float M2 = __shfl_down_sync(kAll, M, d), K2 = __shfl_down_sync(kAll, Kc, d);
        if (lane + d < 32) {
            Kc = fmaf(M, K2, Kc);
            M *= M2;
        }
    }
    float x = __shfl_down_sync(kAll, Kc, 1);   // gh at the next lane's first token
    if (lane == 31) x = 0.f;
    float gh[K];
#pragma unroll
    for (int j = K - 1; j >= 0; --j) {
        if (j < nt) x = fmaf(a_next(j), x, sv[t0 + j]);
        gh[j] = x;
    }
    // Rect, backward: suffix sums
    float seg = 0.f;
#pragma unroll
    for (int j = 0; j < K; ++j)
        if (j < nt) seg += srw[t0 + j] - scl[t0 + j];
    float suf = seg;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const float dn = __shfl_down_sync(kAll, suf, d);
        if (lane + d < 32) suf += dn;
    }
    float r = __shfl_down_sync(kAll, suf, 1);   // the later lanes' sum
    if (lane == 31) r = 0.f;
    float rect[K];
#pragma unroll
    for (int j = K - 1; j >= 0; --j) {
        if (j < nt) r += srw[t0 + j] - scl[t0 + j];
        rect[j] = r;
    }
    // E, forward: this lane's map from E before its first token to E after
    // its last, composed with the maps of the earlier lanes
    float Nm = 1.f, Pm = 0.f;
#pragma unroll
    for (int j = 0; j < K; ++j) {
        if (j < nt) {
            Pm = fmaf(av[j], Pm, dtv[j] * su[t0 + j]);
            Nm *= av[j];
        }
    }
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const float N2 = __shfl_up_sync(kAll, Nm, d), P2 = __shfl_up_sync(kAll, Pm, d);
        if (lane >= d) {
            Pm = fmaf(Nm, P2, Pm);
            Nm *= N2;
        }
    }
    float E = __shfl_up_sync(kAll, Pm, 1);   // E before this lane's first token
    if (lane == 0) E = 0.f;
    float dA = 0.f;
#pragma unroll
    for (int j = 0; j < K; ++j) {
        if (j < nt) {
            const int t = t0 + j;
            const float am1 = j > 0 ? acum[j - 1] : before;
            const float dl = expf(acum[j]) * gh[j] + rect[j] + eAc0 + expf(Ae - am1) * E;
            a.ddt[((size_t)b * a.L + cs.s0 + t) * a.H + h] = sq[t] + Ah * dl;
            dA = fmaf(dtv[j], dl, dA);
            E = fmaf(av[j], E, dtv[j] * su[t]);
        }
    }
    dA = warp_sum(dA);
    if (lane == 0) a.dApart[bhc] = dA;
}

// dB, dC [B,L,G,N] summed over the heads of each group (dC plus dC_add when
// given); dA summed over (b, c) in a fixed order.
__global__ void scan_bwd_reduce(ScanBwdArgs a, int N, int C) {
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
        for (int bb = 0; bb < a.B; ++bb)
            for (int c = 0; c < C; ++c) s += a.dApart[((size_t)bb * a.H + i) * C + c];
        a.dA[i] = s;
    }
}

template <int N, int P>
size_t walk_smem(int S) {
    constexpr int NW = N * P / kCols / 32;
    return sizeof(float) * (kTT * (2 * N + 2 * P) + kTT + 2 * NW * (P + 2) + 2 * S + (size_t)S * NW + NW);
}

template <typename T, int N, int P>
cudaError_t run(const ScanBwdArgs& a, cudaStream_t st) {
    constexpr int NT = N * P / kCols;
    const int C = (a.L + a.S - 1) / a.S;
    const dim3 grid(C, a.H, a.B);
    const bool tc = scan_bwd_tc_applicable(N, P, a.S, std::is_same<T, __nv_bfloat16>::value ? DART_BF16 : DART_F32);
    cudaError_t e;
    if (tc) {
        if ((e = launch_scan_bwd_dS_tc(a, st)) != cudaSuccess) return e;
    } else {
        const size_t smem = sizeof(float) * (kTT * (N + P) + kTT);
        scan_bwd_chunk_adjoint<T, N, P><<<grid, NT, smem, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        const size_t n = (size_t)a.B * a.H * N * P;
        scan_bwd_gin_pass<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a, C);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (tc) {
        // the intra-chunk products on the tensor cores, then the per-token recursions
        if ((e = launch_scan_bwd_quad_tc(a, st)) != cudaSuccess) return e;
        scan_bwd_scalars<<<grid, 32, 0, st>>>(a, C);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    } else {
    {
        const size_t smem = sizeof(float) * RectSmem<N, P>::floats;
        auto k = scan_bwd_rect<T, N, P>;
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return e;
        k<<<grid, 256, smem, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        const size_t smem = walk_smem<N, P>(a.S);
        auto k = scan_bwd_walk<T, N, P>;
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return e;
        k<<<grid, NT, smem, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    }
    const size_t n = (size_t)a.B * a.L * a.G * N;
    const size_t m = n > (size_t)a.H ? n : (size_t)a.H;
    scan_bwd_reduce<<<(unsigned)((m + 255) / 256), 256, 0, st>>>(a, N, C);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launches(5);
    return cudaSuccess;
}

size_t pad256(size_t bytes) { return (bytes + 255) & ~size_t(255); }

}  // namespace

size_t scan_bwd_workspace_bytes(int B, int L, int H, int N, int P, int S) {
    if (B <= 0 || L <= 0 || H <= 0 || N <= 0 || P <= 0 || S <= 0) return 0;
    const size_t C = ((size_t)L + S - 1) / S;
    return pad256(sizeof(float) * B * H * C * N * P)    // dS, then Gin, per chunk
           + pad256(sizeof(float) * B * H * C)          // Ae per chunk
           + pad256(sizeof(float) * 6 * B * H * C * S)  // per-token scalars (Rect alone on CUDA cores)
           + pad256(sizeof(float) * B * H * C)          // sum(Gin o h_in) per chunk
           + 2 * pad256(sizeof(float) * B * L * H * N)  // dB, dC per head
           + pad256(sizeof(float) * B * H * C);         // dA per (b, h, c)
}

bool scan_bwd_supported(int N, int P, int S) {
    const bool np = (N == 128 && P == 64) || (N == 64 && P == 64) || (N == 16 && P == 16);
    return np && S >= 1 && S <= 256;
}

cudaError_t launch_ssd_scan_bwd(ScanBwdArgs a, void* workspace, dart_dtype dt, cudaStream_t st) {
    const size_t C = ((size_t)a.L + a.S - 1) / a.S;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    a.gin = reinterpret_cast<float*>(w);
    w += pad256(sizeof(float) * a.B * a.H * C * a.N * a.P);
    a.asum = reinterpret_cast<float*>(w);
    w += pad256(sizeof(float) * a.B * a.H * C);
    a.rect = reinterpret_cast<float*>(w);
    w += pad256(sizeof(float) * 6 * a.B * a.H * C * a.S);
    a.c0 = reinterpret_cast<float*>(w);
    w += pad256(sizeof(float) * a.B * a.H * C);
    a.dBh = reinterpret_cast<float*>(w);
    w += pad256(sizeof(float) * a.B * a.L * a.H * a.N);
    a.dCh = reinterpret_cast<float*>(w);
    w += pad256(sizeof(float) * a.B * a.L * a.H * a.N);
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
