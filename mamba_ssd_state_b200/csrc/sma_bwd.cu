// sma_bwd.cu -- gradients of state-memory attention with the gated residual
// (the training pass the DART abstract claims; SMA Eqs. (5)-(10), Pith review
// of DART "Core claim" / "What carries the argument"), on CUDA cores.
//
// Forward, per token t of chunk k(t) and memory c < k(t) (raw memories):
//   w1 = dH[c] E_t (N),  s_c = Q_t . w1 / sqrt(N),  v_c = C_t^T dH[c] (P),
//   p = softmax_c(s),  o_t = sum_c p_c v_c,  y_t = y_ssd_t + g o_t.
// Backward of sum(dy * y), with do = g dy_t and D_t = do . o_t:
//   dp_c = do . v_c = C_t . w2,  w2 = dH[c] do (N);   ds_c = p_c (dp_c - D_t)
//   dQ_t = sum_c ds_c w1 / sqrt(N)          dE_t = sum_c ds_c (Q_t^T dH[c]) / sqrt(N)
//   dC_t = sum_h sum_c p_c w2               dg   = sum dy . o
//   ddH[c] = sum_{t: k(t) > c} ( ds_tc / sqrt(N) Q_t E_t^T + p_tc C_t do_t^T )
//
// sma_bwd_rows     grid (tiles of 32 tokens, H, B), 4 threads per token.
//   pass 1 (each thread P/4 value columns): the forward softmax statistics
//     m, l and o_t, recomputed from the memories (not stored by the forward);
//   pass 2 (each thread N/4 state rows): w1, w2 per memory, hence s_c, dp_c,
//     p_c and ds_c; dQ and the head's dC; p and ds go to the workspace;
//   pass 3 (P/4 columns again): Q^T dH[c] per memory, hence dE.
// sma_bwd_memories grid (C, H, B): ddH[c] as an N x P accumulation over the
//   tokens that attend to c, 32 tokens per shared-memory tile.
// sma_bwd_reduce_dc / sma_bwd_reduce_dg: the sums over heads of dC and over
//   tiles of dg, in a fixed order (deterministic).
// Memories are staged in shared memory once per (tile, memory) and shared by
// the tile's 32 tokens.
#include "dart_backward.cuh"

namespace dart {
namespace {

constexpr int kTQ = 32;              // tokens per tile
constexpr int kRowThreads = 4 * kTQ;  // 4 threads per token

template <typename T, int N, int P>
__global__ void __launch_bounds__(kRowThreads) sma_bwd_rows(SmaBwdArgs a) {
    constexpr int PT = P / 4, NT = N / 4;
    constexpr int NS = N + 4, PS = P + 4;   // padded strides (keep 16-byte alignment)
    const int S = a.S, L = a.L, H = a.H, C = (L + S - 1) / S;
    const int t0 = blockIdx.x * kTQ, h = blockIdx.y, b = blockIdx.z;
    const int k = t0 / S;                    // chunk of every token of the tile
    extern __shared__ __align__(16) float sm[];
    float* Qs = sm;                          // [kTQ][NS]
    float* Cs = Qs + kTQ * NS;               // [kTQ][NS]
    float* Es = Cs + kTQ * NS;               // [kTQ][PS]
    float* Ds = Es + kTQ * PS;               // [kTQ][PS]  do = g dy
    float* Ms = Ds + kTQ * PS;               // [N][P]     the memory being read
    const T* Q = static_cast<const T*>(a.Q);
    const T* E = static_cast<const T*>(a.E);
    const T* Cm = static_cast<const T*>(a.Cm);
    const T* dH = static_cast<const T*>(a.dH);
    const float rsn = rsqrtf((float)N);
    const int tl = threadIdx.x / 4, q4 = threadIdx.x % 4;
    const int t = t0 + tl;
    const bool live = t < L;
    const size_t bh = (size_t)b * H + h;

    for (int i = threadIdx.x; i < kTQ * N; i += blockDim.x) {
        const int r = i / N, n = i % N;
        const bool in = t0 + r < L;
        const size_t tok = (size_t)b * L + t0 + r;
        Qs[r * NS + n] = in ? ldf(Q + (tok * H + h) * N + n) : 0.f;
        Cs[r * NS + n] = in ? ldf(Cm + (tok * a.G + group_of(h, H, a.G)) * N + n) : 0.f;
    }
    for (int i = threadIdx.x; i < kTQ * P; i += blockDim.x) {
        const int r = i / P, p = i % P;
        const bool in = t0 + r < L;
        const size_t tok = (size_t)b * L + t0 + r;
        Es[r * PS + p] = in ? ldf(E + (tok * H + h) * P + p) : 0.f;
        Ds[r * PS + p] = in ? a.g * a.dy[(tok * H + h) * P + p] : 0.f;
    }
    const T* mem = dH + bh * (size_t)C * N * P;
    auto stage = [&](int c) {
        __syncthreads();
        for (int i = threadIdx.x; i < N * P; i += blockDim.x) Ms[i] = ldf(mem + (size_t)c * N * P + i);
        __syncthreads();
    };

    // ---- pass 1: m, l, o (this thread's P/4 columns) ----------------------
    float m = -INFINITY, l = 0.f, o[PT];
#pragma unroll
    for (int j = 0; j < PT; ++j) o[j] = 0.f;
    for (int c = 0; c < k; ++c) {
        stage(c);
        float u[PT], v[PT];
#pragma unroll
        for (int j = 0; j < PT; ++j) u[j] = v[j] = 0.f;
        for (int n = 0; n < N; ++n) {
            const float qn = Qs[tl * NS + n], cn = Cs[tl * NS + n];
            const float* row = Ms + n * P + q4 * PT;
#pragma unroll
            for (int j = 0; j < PT; ++j) {
                u[j] = fmaf(qn, row[j], u[j]);
                v[j] = fmaf(cn, row[j], v[j]);
            }
        }
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < PT; ++j) s = fmaf(u[j], Es[tl * PS + q4 * PT + j], s);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s *= kLog2e * rsn;                   // base-2 score
        const float mnew = fmaxf(m, s);
        const float alpha = exp2f(m - mnew), w = exp2f(s - mnew);
        l = l * alpha + w;
#pragma unroll
        for (int j = 0; j < PT; ++j) o[j] = fmaf(o[j], alpha, w * v[j]);
        m = mnew;
    }
    const float inv_l = k > 0 ? 1.f / l : 0.f;
    float Dt = 0.f, dgp = 0.f;
#pragma unroll
    for (int j = 0; j < PT; ++j) {
        o[j] *= inv_l;
        Dt = fmaf(Ds[tl * PS + q4 * PT + j], o[j], Dt);
        if (live) dgp = fmaf(a.dy[(((size_t)b * L + t) * H + h) * P + q4 * PT + j], o[j], dgp);
    }
    Dt += __shfl_xor_sync(0xffffffffu, Dt, 1);
    Dt += __shfl_xor_sync(0xffffffffu, Dt, 2);

    // ---- pass 2: p, ds; dQ and dC (this thread's N/4 rows) -----------------
    float dq[NT], dc[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) dq[j] = dc[j] = 0.f;
    float* pw = a.pbuf + (bh * L + (live ? t : 0)) * (size_t)C;
    float* dsw = a.dsbuf + (bh * L + (live ? t : 0)) * (size_t)C;
    for (int c = 0; c < k; ++c) {
        stage(c);
        float w1[NT], w2[NT];
        float sp = 0.f, dpp = 0.f;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int n = q4 * NT + j;
            const float* row = Ms + n * P;
            float x1 = 0.f, x2 = 0.f;
            for (int p = 0; p < P; ++p) {
                x1 = fmaf(row[p], Es[tl * PS + p], x1);
                x2 = fmaf(row[p], Ds[tl * PS + p], x2);
            }
            w1[j] = x1;
            w2[j] = x2;
            sp = fmaf(Qs[tl * NS + n], x1, sp);
            dpp = fmaf(Cs[tl * NS + n], x2, dpp);
        }
        sp += __shfl_xor_sync(0xffffffffu, sp, 1);
        sp += __shfl_xor_sync(0xffffffffu, sp, 2);
        dpp += __shfl_xor_sync(0xffffffffu, dpp, 1);
        dpp += __shfl_xor_sync(0xffffffffu, dpp, 2);
        const float pc = exp2f(sp * kLog2e * rsn - m) * inv_l;
        const float dsc = pc * (dpp - Dt);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            dq[j] = fmaf(dsc * rsn, w1[j], dq[j]);
            dc[j] = fmaf(pc, w2[j], dc[j]);
        }
        if (live && q4 == 0) {
            pw[c] = pc;
            dsw[c] = dsc;
        }
    }
    if (live) {
        const size_t tok = (size_t)b * L + t;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int n = q4 * NT + j;
            a.dQ[(tok * H + h) * N + n] = dq[j];
            a.dCh[(tok * H + h) * N + n] = dc[j];
        }
    }
    __syncthreads();   // ds of every token of the tile is in the workspace

    // ---- pass 3: dE (this thread's P/4 columns) ----------------------------
    float de[PT];
#pragma unroll
    for (int j = 0; j < PT; ++j) de[j] = 0.f;
    for (int c = 0; c < k; ++c) {
        stage(c);
        const float dsc = live ? dsw[c] * rsn : 0.f;
        float u[PT];
#pragma unroll
        for (int j = 0; j < PT; ++j) u[j] = 0.f;
        for (int n = 0; n < N; ++n) {
            const float qn = Qs[tl * NS + n];
            const float* row = Ms + n * P + q4 * PT;
#pragma unroll
            for (int j = 0; j < PT; ++j) u[j] = fmaf(qn, row[j], u[j]);
        }
#pragma unroll
        for (int j = 0; j < PT; ++j) de[j] = fmaf(dsc, u[j], de[j]);
    }
    if (live) {
        const size_t tok = (size_t)b * L + t;
#pragma unroll
        for (int j = 0; j < PT; ++j) a.dE[(tok * H + h) * P + q4 * PT + j] = de[j];
    }

    // ---- this tile's share of dg, summed in a fixed order -------------------
    __syncthreads();
    float* red = Ms;   // reuse
    red[threadIdx.x] = dgp;
    __syncthreads();
    if (threadIdx.x == 0) {
        float sum = 0.f;
        for (int i = 0; i < kRowThreads; ++i) sum += red[i];
        a.gpart[(bh * gridDim.x) + blockIdx.x] = sum;
    }
}

// ddH[b,h,c] = sum over tokens t with k(t) > c of
//   (ds_tc / sqrt(N)) Q_t E_t^T + p_tc C_t (g dy_t)^T.
// Thread i owns row n = i / (P / CPT) and CPT consecutive columns.
template <typename T, int N, int P>
__global__ void __launch_bounds__(256) sma_bwd_memories(SmaBwdArgs a) {
    constexpr int CPT = N * P / 256;          // columns per thread
    static_assert(N * P % 256 == 0 && P % CPT == 0, "N x P split over 256 threads");
    constexpr int TT = 32;                    // tokens per shared-memory tile
    const int S = a.S, L = a.L, H = a.H, C = (L + S - 1) / S;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    extern __shared__ __align__(16) float sm[];
    float* Qs = sm;                           // [TT][N]
    float* Cs = Qs + TT * N;                  // [TT][N]
    float* Es = Cs + TT * N;                  // [TT][P]
    float* Ds = Es + TT * P;                  // [TT][P]
    float* ws = Ds + TT * P;                  // [TT][2]: ds / sqrt(N), p
    const T* Q = static_cast<const T*>(a.Q);
    const T* E = static_cast<const T*>(a.E);
    const T* Cm = static_cast<const T*>(a.Cm);
    const float rsn = rsqrtf((float)N);
    const int n = threadIdx.x / (P / CPT), p0 = (threadIdx.x % (P / CPT)) * CPT;
    const size_t bh = (size_t)b * H + h;
    float acc[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) acc[j] = 0.f;
    for (int tb = (c + 1) * S; tb < L; tb += TT) {
        __syncthreads();
        for (int i = threadIdx.x; i < TT * N; i += blockDim.x) {
            const int r = i / N, nn = i % N;
            const bool in = tb + r < L;
            const size_t tok = (size_t)b * L + tb + r;
            Qs[i] = in ? ldf(Q + (tok * H + h) * N + nn) : 0.f;
            Cs[i] = in ? ldf(Cm + (tok * a.G + group_of(h, H, a.G)) * N + nn) : 0.f;
        }
        for (int i = threadIdx.x; i < TT * P; i += blockDim.x) {
            const int r = i / P, pp = i % P;
            const bool in = tb + r < L;
            const size_t tok = (size_t)b * L + tb + r;
            Es[i] = in ? ldf(E + (tok * H + h) * P + pp) : 0.f;
            Ds[i] = in ? a.g * a.dy[(tok * H + h) * P + pp] : 0.f;
        }
        for (int r = threadIdx.x; r < TT; r += blockDim.x) {
            const bool in = tb + r < L;
            const size_t row = (bh * L + (in ? tb + r : 0)) * (size_t)C + c;
            ws[2 * r] = in ? a.dsbuf[row] * rsn : 0.f;
            ws[2 * r + 1] = in ? a.pbuf[row] : 0.f;
        }
        __syncthreads();
        for (int r = 0; r < TT; ++r) {
            const float x1 = ws[2 * r] * Qs[r * N + n], x2 = ws[2 * r + 1] * Cs[r * N + n];
#pragma unroll
            for (int j = 0; j < CPT; ++j) acc[j] = fmaf(x1, Es[r * P + p0 + j], fmaf(x2, Ds[r * P + p0 + j], acc[j]));
        }
    }
    float* out = a.ddH + ((bh * C + c) * N + n) * (size_t)P + p0;
#pragma unroll
    for (int j = 0; j < CPT; ++j) out[j] = acc[j];
}

// dC [B,L,G,N]: the per-head parts summed over the heads of each group
__global__ void sma_bwd_reduce_dc(SmaBwdArgs a, int N) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;   // over B * L * G * N
    if (i >= (size_t)a.B * a.L * a.G * N) return;
    const size_t tok = i / ((size_t)a.G * N), n = i % N;
    const int g = (int)((i / N) % a.G), hg = a.H / a.G;
    float sum = 0.f;
    for (int h = g * hg; h < (g + 1) * hg; ++h) sum += a.dCh[(tok * a.H + h) * N + n];
    a.dCm[i] = sum;
}

// dg = the sum of the tile partials: 256 threads each sum a fixed strided
// subset, then a fixed tree (the same order on every run).
__global__ void __launch_bounds__(256) sma_bwd_reduce_dg(SmaBwdArgs a, int nparts) {
    __shared__ float part[256];
    float sum = 0.f;
    for (int i = threadIdx.x; i < nparts; i += 256) sum += a.gpart[i];
    part[threadIdx.x] = sum;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) a.dg[0] = part[0];
}

template <typename T, int N, int P>
cudaError_t run(const SmaBwdArgs& a, cudaStream_t st) {
    const int tiles = (a.L + kTQ - 1) / kTQ;
    const size_t smem_rows = sizeof(float) * (2 * kTQ * (N + 4) + 2 * kTQ * (P + 4) + N * P);
    auto k1 = sma_bwd_rows<T, N, P>;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_rows);
    if (e != cudaSuccess) return e;
    k1<<<dim3(tiles, a.H, a.B), kRowThreads, smem_rows, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int C = (a.L + a.S - 1) / a.S;
    const size_t smem_mem = sizeof(float) * (32 * (2 * N + 2 * P) + 64);
    auto k2 = sma_bwd_memories<T, N, P>;
    if ((e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_mem)) != cudaSuccess)
        return e;
    k2<<<dim3(C, a.H, a.B), 256, smem_mem, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t ndc = (size_t)a.B * a.L * a.G * N;
    sma_bwd_reduce_dc<<<(unsigned)((ndc + 255) / 256), 256, 0, st>>>(a, N);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    sma_bwd_reduce_dg<<<1, 256, 0, st>>>(a, a.B * a.H * tiles);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launches(4);
    return cudaSuccess;
}

}  // namespace

size_t sma_bwd_workspace_bytes(int B, int L, int H, int N, int S) {
    if (B <= 0 || L <= 0 || H <= 0 || N <= 0 || S <= 0) return 0;
    const size_t C = (size_t)(L + S - 1) / S;
    // dg partials: one per 32-token tile (CUDA cores) or per 128-token tile of every chunk (tensor cores)
    size_t tiles = (size_t)(L + kTQ - 1) / kTQ;
    if (S % 128 == 0 && C * (size_t)(S / 128) > tiles) tiles = C * (size_t)(S / 128);
    auto pad = [](size_t bytes) { return (bytes + 255) & ~size_t(255); };
    return 2 * pad(sizeof(float) * B * H * L * C)          // p, ds per (token, memory)
           + pad(sizeof(float) * B * L * H * N)            // dC per head
           + pad(sizeof(float) * B * H * tiles);           // dg per tile
}

cudaError_t launch_sma_bwd(SmaBwdArgs a, void* workspace, dart_dtype dt, cudaStream_t st) {
    const size_t C = (size_t)(a.L + a.S - 1) / a.S;
    auto pad = [](size_t bytes) { return (bytes + 255) & ~size_t(255); };
    uint8_t* w = static_cast<uint8_t*>(workspace);
    a.pbuf = reinterpret_cast<float*>(w);
    w += pad(sizeof(float) * a.B * a.H * a.L * C);
    a.dsbuf = reinterpret_cast<float*>(w);
    w += pad(sizeof(float) * a.B * a.H * a.L * C);
    a.dCh = reinterpret_cast<float*>(w);
    w += pad(sizeof(float) * a.B * a.L * a.H * a.N);
    a.gpart = reinterpret_cast<float*>(w);
    if (sma_bwd_tc_applicable(a.N, a.P, a.S, dt)) {
        // tensor cores: p and ds in [B,H,C,L]; dC per head and dg per tile reduced as below
        cudaError_t e = launch_sma_bwd_tc(a, st);
        if (e != cudaSuccess) return e;
        const size_t ndc = (size_t)a.B * a.L * a.G * a.N;
        sma_bwd_reduce_dc<<<(unsigned)((ndc + 255) / 256), 256, 0, st>>>(a, a.N);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        sma_bwd_reduce_dg<<<1, 256, 0, st>>>(a, sma_bwd_tc_tiles(a.B, a.L, a.H, a.S));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launches(2);
        return cudaSuccess;
    }
#define DART_SMA_BWD_CASE(NN, PP)                                                    \
    if (a.N == NN && a.P == PP)                                                      \
        return dt == DART_F32 ? run<float, NN, PP>(a, st) : run<__nv_bfloat16, NN, PP>(a, st);
    DART_SMA_BWD_CASE(16, 16)
    DART_SMA_BWD_CASE(64, 64)
    DART_SMA_BWD_CASE(128, 64)
#undef DART_SMA_BWD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace dart
