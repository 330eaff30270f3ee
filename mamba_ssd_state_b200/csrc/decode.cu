// decode.cu -- one DART decode step: recurrent update, SSM readout and
// state-memory attention over the cache of chunk memories.
//
// The cache is the length-dependent part of DART's inference state (DART
// abstract; Pith review, "If this is right": N/(2S) of a token-level KV cache,
// Eq. (14)).  A step streams every cached memory once, so the kernel is bound
// by HBM bandwidth: each warp reads whole memories with coalesced 16-byte
// non-allocating loads and reduces with warp shuffles; nothing goes through
// shared memory on the streaming path.
//
// decode_partial  grid (split, h, b), 4 warps.  Split j owns
//   - rows [j*N/ns, (j+1)*N/ns) of the state and of dH_cur: updates them,
//     appends them to the cache when the token closes its chunk, and forms
//     their part of y_ssd = state^T C;
//   - cached memories c in [j*cps, (j+1)*cps) with c < n: per memory
//     v = C^T dH[c], s = (Q^T dH[c]) . E / sqrt(N), merged into one online
//     softmax per block.
//   Writes (m, l, o[P], y_ssd part[P]) for the split to the workspace.
// decode_combine  grid (h, b): merges the splits, y = y_ssd + g * o.
// decode_advance  one thread per sequence: advances (n_chunks, pos) after
//   every block of the step has read them.
//
// E4M3 cache (decode_partial_e4m3): each memory row of P values is stored as
// OCP FP8 E4M3 codes times 2^k (k an int8 per row; the cache quantization
// the pages list as an extension), half the bytes of bf16.  Each lane loads
// 8 codes of a row (8 bytes; four lanes per 32-byte row segment keep the
// warp's loads contiguous) and widens each pair of codes exactly with the
// hardware E4M3x2 -> f16x2 conversion, then to fp32 (every E4M3 value,
// subnormals included, is an f16 value); the products run as packed fp32x2
// FMAs.  The row's 2^k is folded into per-row factors kept in shared memory
// per warp: (q, C) by 2^(k+60), E pre-scaled by 2^-60 for the score and the
// value sum scaled back by 2^-60, so no intermediate overflows for
// contributions up to 2^68 and only contributions below 2^-66 lose bits.  An append
// quantizes the finished memory row by row (one warp per row): the row
// exponent is the smallest k with max|row| 2^-k <= 448 (clamped to
// [-126, 60]) and the codes round to nearest even with saturation.
//
// Decayed memories (memlog set; referee comment 3 on SMA Eq. (8)): memory c
// carries lw = sum_{r=e(c)+1}^{t-1} dt_r A_h.  The warp that reads memory c
// adds this token's dt_t A_h, scales the score by w = exp(lw) and the value
// weight by w, and stores the new lw; a memory appended by this token starts
// at 0 (written by split 0).
#include <cuda_fp8.h>

#include <atomic>

#include "dart_common.cuh"

namespace dart {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kChunksPerSplit = 16;

struct SeqCounters {
    int n, pos;
    bool ok, append;
};

__device__ __forceinline__ SeqCounters read_counters(const DecodeArgs& a, int b) {
    SeqCounters s;
    s.n = a.nchunks[b];
    s.pos = a.pos[b];
    s.ok = s.n >= 0 && s.n <= a.cmax && s.pos >= 0 && s.pos < a.S;
    s.append = s.ok && s.pos == a.S - 1;
    if (s.append && s.n >= a.cmax) s.ok = false;
    return s;
}

template <typename T, int N, int P, bool kDecay>
__global__ void __launch_bounds__(kThreads) decode_partial_kernel(DecodeArgs a) {
    constexpr int VEC = Vec16<T>::kN;        // elements per 16-byte load
    constexpr int LPR = P / VEC;             // lanes per memory row
    constexpr int RPW = 32 / LPR;            // rows per warp load
    static_assert(32 % LPR == 0 && N % RPW == 0, "unsupported (N, P) for decode");
    constexpr int STRIDE = 2 + 2 * P;

    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int ns = gridDim.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const SeqCounters sc = read_counters(a, b);
    float* part = a.part + (((size_t)b * a.H + h) * ns + split) * STRIDE;
    if (!sc.ok) {
        if (split == 0 && h == 0 && tid == 0) flag_status(a.status, kStatusDevice);
        return;
    }
    __shared__ float q_s[N], c_s[N], x_s[P];
    __shared__ float red_m[kWarps], red_l[kWarps], red_o[kWarps][P];
    __shared__ float ypart[kThreads];

    const size_t bh = (size_t)b * a.H + h;
    const T* xt = static_cast<const T*>(a.x) + bh * P;
    const size_t bg = (size_t)b * a.G + group_of(h, a.H, a.G);   // B_t, C_t are [B, G, N]
    const T* Bt = static_cast<const T*>(a.Bm) + bg * N;
    const T* Ct = static_cast<const T*>(a.Cm) + bg * N;
    const T* Qt = static_cast<const T*>(a.Q) + bh * N;
    const T* Et = static_cast<const T*>(a.E) + bh * P;
    const float qscale = kLog2e * rsqrtf((float)N);
    for (int i = tid; i < N; i += kThreads) {
        q_s[i] = qscale * ldf(Qt + i);
        c_s[i] = ldf(Ct + i);
    }
    for (int i = tid; i < P; i += kThreads) x_s[i] = ldf(xt + i);
    __syncthreads();

    // ---- recurrent update of this split's rows --------------------------
    {
        const float dt = a.dt[bh];
        const float decay = expf(dt * a.A[h]);
        const int r0 = split * N / ns, r1 = (split + 1) * N / ns;
        float* st = a.state + bh * N * P;
        float* dc = a.dHcur + bh * N * P;
        T* slot = static_cast<T*>(a.cache) + (bh * a.cmax + sc.n) * (size_t)N * P;
        float yp = 0.f;  // thread owns column p = tid % P when P divides kThreads
        for (int i = r0 * P + tid; i < r1 * P; i += kThreads) {
            const int n = i / P, p = i % P;
            const float inp = dt * ldf(Bt + n) * x_s[p];
            const float hv = fmaf(decay, st[i], inp);
            const float dv = fmaf(decay, dc[i], inp);
            st[i] = hv;
            if (sc.append) {
                slot[i] = Elem<T>::from_f(dv);
                dc[i] = 0.f;
            } else {
                dc[i] = dv;
            }
            yp = fmaf(c_s[n], hv, yp);
        }
        ypart[tid] = yp;
    }

    // ---- state-memory attention over this split's cached chunks ----------
    const int lrow = lane / LPR;             // row inside a warp load
    const int pcol = (lane % LPR) * VEC;     // first column of this lane
    float ev[VEC];
    {
        float tmp[VEC];
#pragma unroll
        for (int j = 0; j < VEC; ++j) tmp[j] = ldf(Et + pcol + j);
#pragma unroll
        for (int j = 0; j < VEC; ++j) ev[j] = tmp[j];
    }
    float m = -INFINITY, l = 0.f, o[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) o[j] = 0.f;
    float* memlog = kDecay ? a.memlog + bh * a.cmax : nullptr;
    const float a_t = kDecay ? a.dt[bh] * a.A[h] : 0.f;   // this token's log-decay
    if (kDecay && sc.append && split == 0 && tid == 0) memlog[sc.n] = 0.f;   // closes at this token
    const int c_begin = split * kChunksPerSplit;
    const int c_end = min(sc.n, c_begin + kChunksPerSplit);
    const T* cache = static_cast<const T*>(a.cache) + bh * a.cmax * (size_t)N * P;
    // decayed memories: lane i holds the log-decay of this warp's i-th memory
    // (memory c_begin + warp + i kWarps), read before and written after the
    // streaming loop so that the loop itself touches only the cache
    static_assert(kChunksPerSplit / kWarps <= 32, "one lane per memory of a warp");
    float lw_mine = 0.f;
    if (kDecay && lane < kChunksPerSplit / kWarps) {
        const int c = c_begin + warp + kWarps * lane;
        if (c < c_end) lw_mine = memlog[c] + a_t;   // now sum_{r=e(c)+1}^{t} dt_r A_h
    }
    int it = 0;   // this warp's memory counter
    for (int c = c_begin + warp; c < c_end; c += kWarps, ++it) {
        const T* mem = cache + (size_t)c * N * P + (size_t)lrow * P + pcol;
        float v[VEC], s = 0.f;
#pragma unroll
        for (int j = 0; j < VEC; ++j) v[j] = 0.f;
        constexpr int ITER = N / RPW;
        constexpr int UNROLL = ITER < 8 ? ITER : 8;
#pragma unroll
        for (int i0 = 0; i0 < ITER; i0 += UNROLL) {
            uint4 raw[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) raw[u] = ld_stream_u4(mem + (size_t)(i0 + u) * RPW * P);
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int n = lrow + (i0 + u) * RPW;
                float mv[VEC];
                if constexpr (VEC == 8) {
                    Vec16<__nv_bfloat16>::unpack(raw[u], mv);
                } else {
                    mv[0] = __uint_as_float(raw[u].x); mv[1] = __uint_as_float(raw[u].y);
                    mv[2] = __uint_as_float(raw[u].z); mv[3] = __uint_as_float(raw[u].w);
                }
                float rd = 0.f;
#pragma unroll
                for (int j = 0; j < VEC; ++j) {
                    v[j] = fmaf(c_s[n], mv[j], v[j]);
                    rd = fmaf(mv[j], ev[j], rd);
                }
                s = fmaf(q_s[n], rd, s);
            }
        }
        // v: sum over lanes holding the same columns; s: sum over the warp
#pragma unroll
        for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
            for (int j = 0; j < VEC; ++j) v[j] += __shfl_xor_sync(0xffffffffu, v[j], off);
        s = warp_sum(s);
        float wd = 1.f;   // decay of memory c at this token (1 for raw memories)
        if (kDecay) {
            wd = exp2f(kLog2e * __shfl_sync(0xffffffffu, lw_mine, it));
            s *= wd;
        }
        const float mnew = fmaxf(m, s);
        const float alpha = exp2f(m - mnew);
        const float w = exp2f(s - mnew);
        l = l * alpha + w;
        const float wv = kDecay ? w * wd : w;
#pragma unroll
        for (int j = 0; j < VEC; ++j) o[j] = fmaf(o[j], alpha, wv * v[j]);
        m = mnew;
    }
    if (kDecay && lane < kChunksPerSplit / kWarps) {
        const int c = c_begin + warp + kWarps * lane;
        if (c < c_end) memlog[c] = lw_mine;
    }
    if (lane == 0) { red_m[warp] = m; red_l[warp] = l; }
    if (lrow == 0) {
#pragma unroll
        for (int j = 0; j < VEC; ++j) red_o[warp][pcol + j] = o[j];
    }
    __syncthreads();
    if (tid < P) {
        float mm = -INFINITY;
        for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, red_m[w]);
        float ll = 0.f, oo = 0.f;
        if (mm != -INFINITY) {
            for (int w = 0; w < kWarps; ++w) {
                const float f = exp2f(red_m[w] - mm);
                ll = fmaf(red_l[w], f, ll);
                oo = fmaf(red_o[w][tid], f, oo);
            }
        }
        float yp = 0.f;
        for (int i = tid; i < kThreads; i += P) yp += ypart[i];
        if (tid == 0) { part[0] = mm; part[1] = ll; }
        part[2 + tid] = oo;
        part[2 + P + tid] = yp;
    }
}

// ---------------------------------------------------------------------------
// E4M3 cache
// ---------------------------------------------------------------------------
// Smallest k with amax 2^-k <= 448 = 0.875 2^9, clamped to [-126, 60].
__device__ __forceinline__ int e4m3_row_exponent(float amax) {
    int e = 0;
    const float f = frexpf(amax, &e);   // amax = f 2^e, f in [0.5, 1); 0 gives f = 0, e = 0
    const int k = f <= 0.875f ? e - 9 : e - 8;
    return min(max(k, -126), 60);
}

// 2^j as an fp32 for j in [-126, 127].
__device__ __forceinline__ float exp2i(int j) { return __int_as_float((j + 127) << 23); }

// Codes 2j and 2j+1 (bytes 2j, 2j+1 of w) as their exact values (x, y).
__device__ __forceinline__ float2 e4m3_pair(uint32_t w, int j) {
    const unsigned short two = (unsigned short)(w >> (16 * j));
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(two));
    return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

// Quantize rows [r0, r1) of a memory from fp32 `src` (row stride P) into
// codes `dst` and exponents `ex`; one warp per row, P / 32 columns per lane.
template <int P>
__device__ __forceinline__ void quantize_rows_e4m3(const float* src, unsigned char* dst, signed char* ex, int r0,
                                                   int r1, int warp, int nwarps, int lane) {
    constexpr int CPL = P / 32;
    static_assert(P % 32 == 0 && CPL <= 4, "E4M3 rows of P values");
    for (int n = r0 + warp; n < r1; n += nwarps) {
        float v[CPL];
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            v[j] = src[(size_t)n * P + lane * CPL + j];
            amax = fmaxf(amax, fabsf(v[j]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const int k = e4m3_row_exponent(amax);
        const float inv = exp2i(-k);   // exact power of two
#pragma unroll
        for (int j = 0; j < CPL; ++j)
            dst[(size_t)n * P + lane * CPL + j] =
                (unsigned char)__nv_cvt_float_to_fp8(v[j] * inv, __NV_SATFINITE, __NV_E4M3);
        if (lane == 0) ex[n] = (signed char)k;
    }
}

// Streaming load of VEC E4M3 codes (8 or 16 bytes) that does not allocate in L1.
template <int VEC> struct CodeLoad;
template <> struct CodeLoad<16> {
    static constexpr int kWords = 4;
    static __device__ __forceinline__ void load(const unsigned char* p, uint32_t* w) {
        const uint4 r = ld_stream_u4(p);
        w[0] = r.x; w[1] = r.y; w[2] = r.z; w[3] = r.w;
    }
};
template <> struct CodeLoad<8> {
    static constexpr int kWords = 2;
    static __device__ __forceinline__ void load(const unsigned char* p, uint32_t* w) {
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "l"(p));
    }
};

#ifndef DART_E4M3_VEC
#define DART_E4M3_VEC 8   // codes per lane per row load (8: measured 500 vs 634 us per step for 16)
#endif
#ifndef DART_E4M3_UNROLL
#define DART_E4M3_UNROLL 8   // row loads in flight per lane
#endif

template <typename T, int N, int P, bool kDecay>
__global__ void __launch_bounds__(kThreads) decode_partial_e4m3_kernel(DecodeArgs a) {
    constexpr int VEC = DART_E4M3_VEC;       // codes per lane load
    constexpr int NW = CodeLoad<VEC>::kWords;
    constexpr int LPR = P / VEC;             // lanes per memory row
    constexpr int RPW = 32 / LPR;            // rows per warp load
    static_assert(32 % LPR == 0 && N % RPW == 0 && N % 32 == 0, "unsupported (N, P) for the E4M3 decode");
    constexpr int STRIDE = 2 + 2 * P;

    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int ns = gridDim.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const SeqCounters sc = read_counters(a, b);
    float* part = a.part + (((size_t)b * a.H + h) * ns + split) * STRIDE;
    if (!sc.ok) {
        if (split == 0 && h == 0 && tid == 0) flag_status(a.status, kStatusDevice);
        return;
    }
    __shared__ float q_s[N], c_s[N], x_s[P];
    __shared__ float2 rowf[kWarps][N];       // per warp: (q_n, C_n) times 2^(k_n + 60) of its current memory
    __shared__ float red_m[kWarps], red_l[kWarps], red_o[kWarps][P];
    __shared__ float ypart[kThreads];

    const size_t bh = (size_t)b * a.H + h;
    const T* xt = static_cast<const T*>(a.x) + bh * P;
    const size_t bg = (size_t)b * a.G + group_of(h, a.H, a.G);   // B_t, C_t are [B, G, N]
    const T* Bt = static_cast<const T*>(a.Bm) + bg * N;
    const T* Ct = static_cast<const T*>(a.Cm) + bg * N;
    const T* Qt = static_cast<const T*>(a.Q) + bh * N;
    const T* Et = static_cast<const T*>(a.E) + bh * P;
    const float qscale = kLog2e * rsqrtf((float)N);
    for (int i = tid; i < N; i += kThreads) {
        q_s[i] = qscale * ldf(Qt + i);
        c_s[i] = ldf(Ct + i);
    }
    for (int i = tid; i < P; i += kThreads) x_s[i] = ldf(xt + i);
    __syncthreads();

    unsigned char* cache8 = static_cast<unsigned char*>(a.cache) + bh * a.cmax * (size_t)N * P;
    signed char* cexp = a.cexp + bh * a.cmax * (size_t)N;
    // ---- recurrent update of this split's rows --------------------------
    const int r0 = split * N / ns, r1 = (split + 1) * N / ns;
    float* dc = a.dHcur + bh * N * P;
    {
        const float dt = a.dt[bh];
        const float decay = expf(dt * a.A[h]);
        float* st = a.state + bh * N * P;
        float yp = 0.f;
        for (int i = r0 * P + tid; i < r1 * P; i += kThreads) {
            const int n = i / P, p = i % P;
            const float inp = dt * ldf(Bt + n) * x_s[p];
            const float hv = fmaf(decay, st[i], inp);
            st[i] = hv;
            dc[i] = fmaf(decay, dc[i], inp);
            yp = fmaf(c_s[n], hv, yp);
        }
        ypart[tid] = yp;
    }
    if (sc.append) {
        // the finished contribution goes to slot n as E4M3 rows, then restarts
        __syncthreads();   // this block's rows of dH_cur are written
        quantize_rows_e4m3<P>(dc, cache8 + (size_t)sc.n * N * P, cexp + (size_t)sc.n * N, r0, r1, warp, kWarps,
                              lane);
        __syncthreads();
        for (int i = r0 * P + tid; i < r1 * P; i += kThreads) dc[i] = 0.f;
    }

    // ---- state-memory attention over this split's cached chunks ----------
    const int lrow = lane / LPR;             // row inside a warp load
    const int pcol = (lane % LPR) * VEC;     // first column of this lane
    constexpr float kTwoM60 = 8.67361737988403547e-19f;   // 2^-60
    float2 ev2[VEC / 2];
#pragma unroll
    for (int j = 0; j < VEC / 2; ++j)
        ev2[j] = make_float2(kTwoM60 * ldf(Et + pcol + 2 * j), kTwoM60 * ldf(Et + pcol + 2 * j + 1));
    float m = -INFINITY, l = 0.f;
    float2 o2[VEC / 2];
#pragma unroll
    for (int j = 0; j < VEC / 2; ++j) o2[j] = make_float2(0.f, 0.f);
    float* memlog = kDecay ? a.memlog + bh * a.cmax : nullptr;
    const float a_t = kDecay ? a.dt[bh] * a.A[h] : 0.f;
    if (kDecay && sc.append && split == 0 && tid == 0) memlog[sc.n] = 0.f;
    const int c_begin = split * kChunksPerSplit;
    const int c_end = min(sc.n, c_begin + kChunksPerSplit);
    static_assert(kChunksPerSplit / kWarps <= 32, "one lane per memory of a warp");
    float lw_mine = 0.f;
    if (kDecay && lane < kChunksPerSplit / kWarps) {
        const int c = c_begin + warp + kWarps * lane;
        if (c < c_end) lw_mine = memlog[c] + a_t;
    }
    float2* rf = rowf[warp];
    int it = 0;
    for (int c = c_begin + warp; c < c_end; c += kWarps, ++it) {
        const unsigned char* mem = cache8 + (size_t)c * N * P + (size_t)lrow * P + pcol;
        // row factors of this memory: (q_n, C_n) 2^(k_n + 60)
        __syncwarp();   // the previous memory's factors are no longer read
#pragma unroll
        for (int n = lane; n < N; n += 32) {
            const float r2 = exp2i((int)cexp[(size_t)c * N + n] + 60);
            rf[n] = make_float2(q_s[n] * r2, c_s[n] * r2);
        }
        __syncwarp();
        float2 v2[VEC / 2];
#pragma unroll
        for (int j = 0; j < VEC / 2; ++j) v2[j] = make_float2(0.f, 0.f);
        float s = 0.f;
        constexpr int ITER = N / RPW;
        constexpr int UNROLL = ITER < DART_E4M3_UNROLL ? ITER : DART_E4M3_UNROLL;
#pragma unroll
        for (int i0 = 0; i0 < ITER; i0 += UNROLL) {
            uint32_t raw[UNROLL][NW];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) CodeLoad<VEC>::load(mem + (size_t)(i0 + u) * RPW * P, raw[u]);
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const float2 f_qc = rf[lrow + (i0 + u) * RPW];
                const float2 cs2 = make_float2(f_qc.y, f_qc.y);
                float2 rd2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int q = 0; q < NW; ++q) {
#pragma unroll
                    for (int i = 0; i < 4; i += 2) {
                        const float2 f = e4m3_pair(raw[u][q], i / 2);
                        v2[2 * q + i / 2] = __ffma2_rn(cs2, f, v2[2 * q + i / 2]);
                        rd2 = __ffma2_rn(f, ev2[2 * q + i / 2], rd2);
                    }
                }
                s = fmaf(f_qc.x, rd2.x + rd2.y, s);
            }
        }
        float v[VEC];
#pragma unroll
        for (int j = 0; j < VEC / 2; ++j) { v[2 * j] = v2[j].x; v[2 * j + 1] = v2[j].y; }
#pragma unroll
        for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
            for (int j = 0; j < VEC; ++j) v[j] += __shfl_xor_sync(0xffffffffu, v[j], off);
        s = warp_sum(s);
        float wd = 1.f;
        if (kDecay) {
            wd = exp2f(kLog2e * __shfl_sync(0xffffffffu, lw_mine, it));
            s *= wd;
        }
        const float mnew = fmaxf(m, s);
        const float alpha = exp2f(m - mnew);
        const float w = exp2f(s - mnew);
        l = l * alpha + w;
        const float wv = (kDecay ? w * wd : w) * kTwoM60;   // the value sum carries 2^60
        const float2 al2 = make_float2(alpha, alpha), wv2 = make_float2(wv, wv);
#pragma unroll
        for (int j = 0; j < VEC / 2; ++j)
            o2[j] = __ffma2_rn(o2[j], al2, __fmul2_rn(wv2, make_float2(v[2 * j], v[2 * j + 1])));
        m = mnew;
    }
    if (kDecay && lane < kChunksPerSplit / kWarps) {
        const int c = c_begin + warp + kWarps * lane;
        if (c < c_end) memlog[c] = lw_mine;
    }
    if (lane == 0) { red_m[warp] = m; red_l[warp] = l; }
    if (lrow == 0) {
#pragma unroll
        for (int j = 0; j < VEC / 2; ++j) {
            red_o[warp][pcol + 2 * j] = o2[j].x;
            red_o[warp][pcol + 2 * j + 1] = o2[j].y;
        }
    }
    __syncthreads();
    if (tid < P) {
        float mm = -INFINITY;
        for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, red_m[w]);
        float ll = 0.f, oo = 0.f;
        if (mm != -INFINITY) {
            for (int w = 0; w < kWarps; ++w) {
                const float f = exp2f(red_m[w] - mm);
                ll = fmaf(red_l[w], f, ll);
                oo = fmaf(red_o[w][tid], f, oo);
            }
        }
        float yp = 0.f;
        for (int i = tid; i < kThreads; i += P) yp += ypart[i];
        if (tid == 0) { part[0] = mm; part[1] = ll; }
        part[2 + tid] = oo;
        part[2 + P + tid] = yp;
    }
}

// Prefill memories -> E4M3 cache slots: one warp per memory row.
template <typename T, int P>
__global__ void __launch_bounds__(256) cache_quantize_e4m3_kernel(int H, int C, int N, int nmem, int cmax,
                                                                   const T* __restrict__ dH,
                                                                   unsigned char* __restrict__ cache,
                                                                   signed char* __restrict__ cexp, long rows) {
    constexpr int CPL = P / 32;
    const long row = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;   // rows = B * H * nmem * N
    const int n = (int)(row % N);
    const long r = row / N;
    const int c = (int)(r % nmem);
    const long bh = r / nmem;
    const T* src = dH + ((bh * C + c) * (long)N + n) * P + lane * CPL;
    float v[CPL];
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        v[j] = ldf(src + j);
        amax = fmaxf(amax, fabsf(v[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int k = e4m3_row_exponent(amax);
    const float inv = exp2i(-k);
    unsigned char* dst = cache + ((bh * cmax + c) * (long)N + n) * P + lane * CPL;
#pragma unroll
    for (int j = 0; j < CPL; ++j) dst[j] = (unsigned char)__nv_cvt_float_to_fp8(v[j] * inv, __NV_SATFINITE, __NV_E4M3);
    if (lane == 0) cexp[(bh * cmax + c) * (long)N + n] = (signed char)k;
}

template <int P>
__global__ void __launch_bounds__(P) decode_combine_kernel(DecodeArgs a) {
    constexpr int STRIDE = 2 + 2 * P;
    const int h = blockIdx.x, b = blockIdx.y, p = threadIdx.x;
    const SeqCounters sc = read_counters(a, b);
    if (!sc.ok) return;
    const int ns = a.nsplit;
    const float* part = a.part + ((size_t)b * a.H + h) * ns * STRIDE;
    float mm = -INFINITY;
    for (int j = 0; j < ns; ++j) mm = fmaxf(mm, part[j * STRIDE]);
    float l = 0.f, o = 0.f, y = 0.f;
    for (int j = 0; j < ns; ++j) {
        const float* pj = part + j * STRIDE;
        if (mm != -INFINITY) {
            const float f = exp2f(pj[0] - mm);
            l = fmaf(pj[1], f, l);
            o = fmaf(pj[2 + p], f, o);
        }
        y += pj[2 + P + p];
    }
    const float oo = l > 0.f ? o / l : 0.f;
    a.y[((size_t)b * a.H + h) * P + p] = fmaf(a.g, oo, y);
}

// Advances the per-sequence counters once every head has read them.
__global__ void decode_advance_kernel(DecodeArgs a) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= a.B) return;
    const SeqCounters sc = read_counters(a, b);
    if (!sc.ok) return;
    if (sc.append) {
        a.nchunks[b] = sc.n + 1;
        a.pos[b] = 0;
    } else {
        a.pos[b] = sc.pos + 1;
    }
}

// One warp per (b, h): suffix sums of dt A over the prefill, walked from the
// last token down 32 tokens at a time with an fp64 carry; the suffix that
// starts at a chunk boundary (c+1) S is memory c's log-decay.
__global__ void __launch_bounds__(256) memlog_init_kernel(int BH, int L, int H, int S, int cmax,
                                                           const float* __restrict__ dt,
                                                           const float* __restrict__ A, float* __restrict__ memlog) {
    const int bh = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (bh >= BH) return;
    const int b = bh / H, h = bh % H;
    const int ncached = L / S;            // complete chunks of the prefill
    float* out = memlog + (size_t)bh * cmax;
    if (lane == 0 && ncached > 0 && ncached * S == L) out[ncached - 1] = 0.f;   // closed at the last token
    const float Ah = A[h];
    double carry = 0.0;
    for (int base = L - 1; base >= S; base -= 32) {
        const int t = base - lane;
        float v = t >= 0 ? dt[((size_t)b * L + t) * H + h] * Ah : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        if (t >= S && t % S == 0) out[t / S - 1] = (float)(carry + (double)v);
        carry += (double)__shfl_sync(0xffffffffu, v, 31);
    }
}

template <typename T, int N, int P>
cudaError_t run(const DecodeArgs& a, cudaStream_t st) {
    if (a.memlog)
        decode_partial_kernel<T, N, P, true><<<dim3(a.nsplit, a.H, a.B), kThreads, 0, st>>>(a);
    else
        decode_partial_kernel<T, N, P, false><<<dim3(a.nsplit, a.H, a.B), kThreads, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine_kernel<P><<<dim3(a.H, a.B), P, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    decode_advance_kernel<<<(a.B + 127) / 128, 128, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launches(3);
    return cudaSuccess;
}

template <typename T, int N, int P>
cudaError_t run_e4m3(const DecodeArgs& a, cudaStream_t st) {
    if (a.memlog)
        decode_partial_e4m3_kernel<T, N, P, true><<<dim3(a.nsplit, a.H, a.B), kThreads, 0, st>>>(a);
    else
        decode_partial_e4m3_kernel<T, N, P, false><<<dim3(a.nsplit, a.H, a.B), kThreads, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine_kernel<P><<<dim3(a.H, a.B), P, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    decode_advance_kernel<<<(a.B + 127) / 128, 128, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launches(3);
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_decode_memlog_init(int B, int L, int H, int S, int cmax, const float* dt, const float* A,
                                      float* memlog, cudaStream_t st) {
    const int BH = B * H;
    memlog_init_kernel<<<(BH + 7) / 8, 256, 0, st>>>(BH, L, H, S, cmax, dt, A, memlog);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaSuccess;
}

bool decode_e4m3_supported(int N, int P) { return P == 64 && (N == 128 || N == 64); }

cudaError_t launch_decode_e4m3(const DecodeArgs& a, dart_dtype dt, cudaStream_t st) {
    if (a.P != 64 || !a.cexp) return cudaErrorInvalidValue;
    if (a.N == 128) return dt == DART_F32 ? run_e4m3<float, 128, 64>(a, st) : run_e4m3<__nv_bfloat16, 128, 64>(a, st);
    if (a.N == 64) return dt == DART_F32 ? run_e4m3<float, 64, 64>(a, st) : run_e4m3<__nv_bfloat16, 64, 64>(a, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_cache_quantize_e4m3(int B, int H, int C, int N, int P, int nmem, int cmax, const void* dH,
                                       dart_dtype dt, unsigned char* cache, signed char* cexp, cudaStream_t st) {
    if (P != 64 || nmem < 0 || nmem > C || nmem > cmax) return cudaErrorInvalidValue;
    const long rows = (long)B * H * nmem * N;
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + 7) / 8);
    if (dt == DART_F32)
        cache_quantize_e4m3_kernel<float, 64><<<grid, 256, 0, st>>>(H, C, N, nmem, cmax,
                                                                    static_cast<const float*>(dH), cache, cexp, rows);
    else
        cache_quantize_e4m3_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(
            H, C, N, nmem, cmax, static_cast<const __nv_bfloat16*>(dH), cache, cexp, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaSuccess;
}

int decode_num_splits(int, int, int cmax) {
    const long long ns = ((long long)cmax + kChunksPerSplit - 1) / kChunksPerSplit;
    return ns < 1 ? 1 : (int)ns;
}

bool decode_supported(int N, int P, int S, dart_dtype) {
    const bool np = (N == 16 && P == 16) || (N == 64 && P == 64) || (N == 128 && P == 64);
    return np && S >= 1;
}

cudaError_t launch_decode(const DecodeArgs& a, dart_dtype dt, cudaStream_t st) {
#define DART_DEC_CASE(NN, PP)                                                       \
    if (a.N == NN && a.P == PP)                                                     \
        return dt == DART_F32 ? run<float, NN, PP>(a, st) : run<__nv_bfloat16, NN, PP>(a, st);
    DART_DEC_CASE(16, 16)
    DART_DEC_CASE(64, 64)
    DART_DEC_CASE(128, 64)
#undef DART_DEC_CASE
    return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// Fixed scratch for dart_decode_step_noalloc.
//
// Callers that cannot allocate device memory get the decode step's split
// partials in this file-scope array instead of a workspace they pass in.  It
// exists once per device that loads the library and lives until the process
// exits.  Every call shares it and it keeps the last call's contents; the
// decode kernels write every slot they later read, so nothing needs clearing.
// Calls that overlap on the GPU (different streams, or different threads
// without ordering) race on it.
//
// On the host `g_noalloc_scratch` names a host-side stand-in, not the device
// array, so kernels are given the address cudaGetSymbolAddress reports for
// the current device.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    // looked up once per device; threads that race on the first lookup store the same value
    static std::atomic<void*> cache[64];
    void* p = cache[dev].load(std::memory_order_relaxed);
    if (!p) {
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        cache[dev].store(p, std::memory_order_relaxed);
    }
    *out = p;
    return cudaSuccess;
}

}  // namespace dart
