// sma_bwd_tc.cu -- gradients of state-memory attention on the 5th-generation
// tensor cores (the training pass the DART abstract claims; SMA Eqs.
// (5)-(10), Pith review of DART "Core claim" / "What carries the argument").
//
// Forward, per token t of chunk k(t) and memory c < k(t):
//   U_c = Q_t^T dH[c], V_c = C_t^T dH[c]  (P),  s_c = U_c . E_t / sqrt(N),
//   p = softmax_c(s),  o_t = sum_c p_c V_c,  y_t = y_ssd_t + g o_t.
// Backward of sum(dy * y), with do = g dy_t and delta_t = do . o_t:
//   dp_c = do . V_c,  ds_c = p_c (dp_c - delta_t),
//   dE_t = sum_c ds_c U_c / sqrt(N)                       (CUDA cores)
//   dQ_t = sum_c (ds_c / sqrt(N)) dH[c] E_t = [(ds/sqrt(N)) E_T] dH[c]^T
//   dC_t = sum_c p_c dH[c] do_t             = [p do_T] dH[c]^T    (per head)
//   ddH[c] = Q^T diag(ds_.c / sqrt(N)) E + C^T diag(p_.c) do   (tokens k(t) > c)
//
// sma_bwd_q_tc   one CTA per 128-token query tile of one (b, h).  Pass 1
//   re-runs the forward over the tile's memories (U, V by tcgen05; scores,
//   online softmax, o on CUDA cores) for the softmax statistics and delta.
//   Pass 2 runs U, V again and, per memory, forms p and ds, accumulates dE
//   in registers, writes the rows of (ds / sqrt(N)) E and p do as bf16
//   K-major tiles and issues dQ += tile x dH[c]^T, dC += tile x dH[c]^T with
//   dH[c] (already in shared memory as the MN-major B of U, V) as a K-major
//   B; dQ and dC accumulate in TMEM over the memories.  p and ds go to the
//   workspace for the memory side.
//   Roles (320 threads): warp 0 TMA, warp 1 TMEM + MMA, warps 2-9 the rows
//   as four pairs (one per TMEM lane quadrant), each warp of a pair 32 of
//   the 64 value columns, partial dot products exchanged in shared memory.
//   TMEM: U, V double-buffered (2 x 128 columns), dQ (128), dC (128).
// sma_bwd_dh_tc  one CTA per pair of chunk memories of one (b, h): over the
//   query tiles of the later chunks, ddH[c] (TMEM, 128 lanes n x 64 columns p) +=
//   Q_T^T x [(ds / sqrt(N)) E_T] + C_T^T x [p do_T], with Q_T and C_T loaded
//   by TMA and used as MN-major A operands, the scaled rows built by four
//   warps as MN-major B operands.
// The tensor-core operands are bf16: Q, C, E, dH as given; the scaled rows
// are rounded to bf16 (2^-9 relative), the products accumulate in fp32.
#include <cuda_bf16.h>
#include <string.h>

#include "dart_backward.cuh"
#include "sm100.cuh"
#include "tensor_map.h"

namespace dart {
namespace {

using namespace sm100;

constexpr int kN = 128, kP = 64;   // compiled shape
constexpr int kBQ = 128;           // query tokens per tile (MMA M)
constexpr uint32_t kPanel = 128 * 64 * 2;   // 128 rows x 64 bf16, one 128-byte swizzle panel
constexpr uint32_t kMem = kN * kP * 2;      // one chunk memory, 16 KB

struct SmaBwdTcParams {
    CUtensorMap tmap_q;  // Q  (N, H, L, B), box (64, 1, 128, 1)
    CUtensorMap tmap_c;  // Cm (N, G, L, B), box (64, 1, 128, 1)
    CUtensorMap tmap_h;  // dH (P, B*H*C*N), box (64, 128)
    const __nv_bfloat16* E;
    const float* dy;
    float g;
    int B, L, H, S, C, HG, tpc;   // tpc: 128-token tiles per chunk
    float* dQ; float* dE; float* dCh; float* ddH;
    float* pbuf; float* dsbuf;    // [B,H,C,L]
    float* gpart;                 // [tiles]
    int* status;
};

// Query tile `i` in order of decreasing chunk index (most memories first).
struct QTile {
    int b, h, k, t0;
};
__device__ __forceinline__ QTile q_tile(const SmaBwdTcParams& p, int i) {
    const int per_k = p.B * p.H * p.tpc;
    QTile t;
    t.k = p.C - 1 - i / per_k;
    const int r = i % per_k, bh = r / p.tpc;
    t.b = bh / p.H;
    t.h = bh % p.H;
    t.t0 = t.k * p.S + (r % p.tpc) * kBQ;
    return t;
}

// Eight bf16 of a row as fp32 (a bf16 is the top half of an fp32).
__device__ __forceinline__ void widen8(uint4 v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}
// 16-byte chunk `q` (8 bf16) of row `r` of a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_chunk(uint32_t base, int r, int q) {
    return base + (uint32_t)r * 128u + ((uint32_t)(q ^ (r & 7)) << 4);
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// ===========================================================================
// query side
// ===========================================================================
namespace qs {
constexpr int kStages = 4;
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffC = 2 * kPanel;
constexpr uint32_t kOffH = 4 * kPanel;
constexpr uint32_t kOffA2 = kOffH + kStages * kMem;   // 2 buffers of (ds / sqrt(N)) E rows
constexpr uint32_t kOffA3 = kOffA2 + 2 * kPanel;      // 2 buffers of p do rows
constexpr uint32_t kOffX = kOffA3 + 2 * kPanel;       // exchange [2 parity][2 half][128 rows] float2
constexpr uint32_t kOffBar = kOffX + 2 * 2 * 128 * 8;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kColDQ = 256, kColDC = 384;
enum Bar { QC_FULL = 0, H_FULL0 = 1, H_EMPTY0 = H_FULL0 + kStages, UV_FULL0 = H_EMPTY0 + kStages,
           UV_EMPTY0 = UV_FULL0 + 2, A_FULL0 = UV_EMPTY0 + 2, A_EMPTY0 = A_FULL0 + 2, D_FULL = A_EMPTY0 + 2,
           NUM_BARS };
static_assert(NUM_BARS * 8 + 16 <= 256 && kSmemBytes <= 232448, "shared memory layout");
}  // namespace qs

__global__ void __launch_bounds__(qs::kThreads, 1) sma_bwd_q_tc(const __grid_constant__ SmaBwdTcParams p) {
    using namespace qs;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffBar + NUM_BARS * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    float* red = reinterpret_cast<float*>(tmem_holder + 2);   // [4] per-quadrant dg partials
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const QTile t = q_tile(p, blockIdx.x);
    const bool active = t.k > 0 && t.t0 < p.L;
    const size_t bh = (size_t)t.b * p.H + t.h;

    if (threadIdx.x == 0) {
        mbar_init(bar(QC_FULL), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(H_FULL0 + s), 1);
            mbar_init(bar(H_EMPTY0 + s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(UV_FULL0 + i), 1);
            mbar_init(bar(UV_EMPTY0 + i), kEpiWarps);
            mbar_init(bar(A_FULL0 + i), kEpiWarps);
            mbar_init(bar(A_EMPTY0 + i), 1);
        }
        mbar_init(bar(D_FULL), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tmap_q);
        tma_prefetch_desc(&p.tmap_c);
        tma_prefetch_desc(&p.tmap_h);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const WaitCtx wc{abort_flag, p.status, 4};

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA
        if (active) {
            bool ok = true;
            if (lane == 0) {
                mbar_expect_tx(bar(QC_FULL), 4 * kPanel);
                tma_load_4d(sbase + kOffQ, &p.tmap_q, bar(QC_FULL), 0, t.h, t.t0, t.b);
                tma_load_4d(sbase + kOffQ + kPanel, &p.tmap_q, bar(QC_FULL), 64, t.h, t.t0, t.b);
                tma_load_4d(sbase + kOffC, &p.tmap_c, bar(QC_FULL), 0, t.h / p.HG, t.t0, t.b);
                tma_load_4d(sbase + kOffC + kPanel, &p.tmap_c, bar(QC_FULL), 64, t.h / p.HG, t.t0, t.b);
            }
            // every memory twice: pass 1, then pass 2
            for (int it = 0; it < 2 * t.k && ok; ++it) {
                const int c = it % t.k, s = it % kStages;
                if (!(ok = mbar_wait_warp(bar(H_EMPTY0 + s), ((uint32_t)(it / kStages) & 1u) ^ 1u, wc, 1))) break;
                if (lane == 0) {
                    mbar_expect_tx(bar(H_FULL0 + s), kMem);
                    tma_load_2d(sbase + kOffH + (uint32_t)s * kMem, &p.tmap_h, bar(H_FULL0 + s), 0,
                                (int)((bh * p.C + c) * kN));
                }
                __syncwarp();
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        if (active) {
            bool ok = mbar_wait_warp(bar(QC_FULL), 0, wc, 2);
            tc_fence_after();
            const uint32_t id_uv = idesc_bf16_f32(kBQ, kP, false, true);    // A K-major, B (dH) MN-major
            const uint32_t id_dq = idesc_bf16_f32(kBQ, kN, false, false);   // A K-major, B (dH) K-major
            int iu = 0;
            // U, V of the memory in ring stage s into buffer iu & 1
            auto mma_uv = [&](int it) -> bool {
                const int s = it % kStages;
                if (!mbar_wait_warp(bar(H_FULL0 + s), (uint32_t)(it / kStages) & 1u, wc, 3)) return false;
                if (!mbar_wait_warp(bar(UV_EMPTY0 + (iu & 1)), ((uint32_t)(iu >> 1) & 1u) ^ 1u, wc, 4)) return false;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t hb = sbase + kOffH + (uint32_t)s * kMem;
                    const uint32_t d = tmem + (uint32_t)(iu & 1) * 128;
#pragma unroll
                    for (int kk = 0; kk < kN / 16; ++kk) {
                        const uint32_t ka = (uint32_t)(kk >> 2) * kPanel + (uint32_t)(kk & 3) * 32;
                        const uint64_t bd = smem_desc_sw128(hb + (uint32_t)kk * 2048, kMem, 1024);
                        mma_f16_ss(d, smem_desc_sw128(sbase + kOffQ + ka, 16, 1024), bd, id_uv, kk > 0 ? 1u : 0u);
                        mma_f16_ss(d + 64, smem_desc_sw128(sbase + kOffC + ka, 16, 1024), bd, id_uv, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(UV_FULL0 + (iu & 1)));
                }
                __syncwarp();
                ++iu;
                return true;
            };
            // pass 1
            for (int c = 0; c < t.k && ok; ++c) {
                if (!(ok = mma_uv(c))) break;
                if (lane == 0) mma_commit(bar(H_EMPTY0 + c % kStages));
                __syncwarp();
            }
            // pass 2: U, V of memory c + 1 go out before dQ, dC of memory c
            if (ok) ok = mma_uv(t.k);
            for (int c = 0; c < t.k && ok; ++c) {
                const int it = t.k + c, s = it % kStages;
                if (c + 1 < t.k && !(ok = mma_uv(it + 1))) break;
                if (!(ok = mbar_wait_warp(bar(A_FULL0 + (c & 1)), (uint32_t)(c >> 1) & 1u, wc, 5))) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t hb = sbase + kOffH + (uint32_t)s * kMem;
                    const uint32_t a2 = sbase + kOffA2 + (uint32_t)(c & 1) * kPanel;
                    const uint32_t a3 = sbase + kOffA3 + (uint32_t)(c & 1) * kPanel;
#pragma unroll
                    for (int kk = 0; kk < kP / 16; ++kk) {
                        const uint64_t bd = smem_desc_sw128(hb + (uint32_t)kk * 32, 16, 1024);
                        const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
                        mma_f16_ss(tmem + kColDQ, smem_desc_sw128(a2 + (uint32_t)kk * 32, 16, 1024), bd, id_dq, acc);
                        mma_f16_ss(tmem + kColDC, smem_desc_sw128(a3 + (uint32_t)kk * 32, 16, 1024), bd, id_dq, acc);
                    }
                    mma_commit(bar(A_EMPTY0 + (c & 1)));
                    mma_commit(bar(H_EMPTY0 + s));
                    if (c == t.k - 1) mma_commit(bar(D_FULL));
                }
                __syncwarp();
            }
        }
    } else {
        // ---------------------------------------------------------- the rows
        const int quad = warp & 3, half = (warp - 2) >> 2, col0 = half * 32;
        const int row = quad * 32 + lane;
        const int tok = t.t0 + row;
        const bool inrow = tok < p.L;
        const size_t orow = ((size_t)t.b * p.L + tok) * p.H + t.h;   // token row of (b, h)
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        const float sscale = kLog2e * rsqrtf((float)kN), inv_sqrt_n = rsqrtf((float)kN);
        float2* xch = reinterpret_cast<float2*>(smem + kOffX);
        auto pair_sync = [&]() { named_bar_sync(2 + quad, 64); };
        if (!active) {
            if (inrow) {   // no memory: every gradient of these rows is zero
                float4* q4 = reinterpret_cast<float4*>(p.dQ + orow * kN + half * 64);
                float4* c4 = reinterpret_cast<float4*>(p.dCh + orow * kN + half * 64);
                float4* e4 = reinterpret_cast<float4*>(p.dE + orow * kP + col0);
                const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int j = 0; j < 16; ++j) q4[j] = c4[j] = z;
#pragma unroll
                for (int j = 0; j < 8; ++j) e4[j] = z;
            }
            if (threadIdx.x == 64) p.gpart[blockIdx.x] = 0.f;
        } else {
            float e[32], dy[32];
            if (inrow) {
                const uint4* es = reinterpret_cast<const uint4*>(p.E + orow * kP + col0);
#pragma unroll
                for (int q = 0; q < 4; ++q) widen8(__ldg(es + q), e + 8 * q);
                const float4* ds4 = reinterpret_cast<const float4*>(p.dy + orow * kP + col0);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 v = __ldg(ds4 + q);
                    dy[4 * q] = v.x; dy[4 * q + 1] = v.y; dy[4 * q + 2] = v.z; dy[4 * q + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) e[j] = dy[j] = 0.f;
            }
            bool ok = true;
            int iu = 0, xi = 0;
            // U and V (this warp's 32 columns) of MMA round iu, then the buffer goes back
            auto load_uv = [&](float* u, float* v) {
                if (ok) ok = mbar_wait_warp(bar(UV_FULL0 + (iu & 1)), (uint32_t)(iu >> 1) & 1u, wc, 6);
                if (ok) {
                    tc_fence_after();
                    const uint32_t col = (uint32_t)(iu & 1) * 128 + (uint32_t)col0;
                    tmem_ld_32x32b_x32(t_lane + col, u);
                    tmem_ld_32x32b_x32(t_lane + col + 64, v);
                    tmem_ld_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(UV_EMPTY0 + (iu & 1)));
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) u[j] = v[j] = 0.f;
                }
                ++iu;
            };
            // (a, b) of this row summed with the partner warp's
            auto exchange = [&](float a, float b) -> float2 {
                xch[((xi & 1) * 2 + half) * 128 + row] = make_float2(a, b);
                pair_sync();
                const float2 o = xch[((xi & 1) * 2 + (1 - half)) * 128 + row];
                ++xi;
                return make_float2(a + o.x, b + o.y);
            };
            // ---- pass 1: softmax statistics and o -------------------------
            float m = -INFINITY, l = 0.f, o[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0.f;
            for (int c = 0; c < t.k; ++c) {
                float u[32], v[32];
                load_uv(u, v);
                float ps = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) ps = fmaf(u[j], e[j], ps);
                const float s = exchange(ps, 0.f).x * sscale;
                const float mn = fmaxf(m, s), alpha = exp2f(m - mn), w = exp2f(s - mn);
                l = l * alpha + w;
#pragma unroll
                for (int j = 0; j < 32; ++j) o[j] = fmaf(w, v[j], o[j] * alpha);
                m = mn;
            }
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            float dyo = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) dyo = fmaf(dy[j], o[j] * inv_l, dyo);
            dyo = exchange(dyo, 0.f).x;                 // dy . o_t over all 64 columns
            const float lse = m + log2f(l > 0.f ? l : 1.f);
            const float delta = p.g * dyo;
            {   // dg partial of the tile: sum over its rows of dy . o
                float r = half == 0 && inrow ? dyo : 0.f;
                r = warp_sum(r);
                if (half == 0 && lane == 0) red[quad] = r;
                named_bar_sync(1, 32 * kEpiWarps);
                if (threadIdx.x == 64) p.gpart[blockIdx.x] = (red[0] + red[1]) + (red[2] + red[3]);
            }
            // ---- pass 2: p, ds; dE; the dQ / dC operand rows --------------
            float de[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) de[j] = 0.f;
            for (int c = 0; c < t.k; ++c) {
                float u[32], v[32];
                load_uv(u, v);
                float ps = 0.f, pd = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    ps = fmaf(u[j], e[j], ps);
                    pd = fmaf(v[j], dy[j], pd);
                }
                const float2 sd = exchange(ps, pd);
                const float pc = inrow ? exp2f(sd.x * sscale - lse) : 0.f;
                const float ds = pc * (p.g * sd.y - delta);
                const float dsn = ds * inv_sqrt_n, pg = pc * p.g;
#pragma unroll
                for (int j = 0; j < 32; ++j) de[j] = fmaf(dsn, u[j], de[j]);
                if (ok) ok = mbar_wait_warp(bar(A_EMPTY0 + (c & 1)), ((uint32_t)(c >> 1) & 1u) ^ 1u, wc, 7);
                if (ok) {
                    const uint32_t a2 = sbase + kOffA2 + (uint32_t)(c & 1) * kPanel;
                    const uint32_t a3 = sbase + kOffA3 + (uint32_t)(c & 1) * kPanel;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int j = 8 * q;
                        st_shared_v4(sw128_chunk(a2, row, 4 * half + q),
                                     make_uint4(pack_bf16(dsn * e[j], dsn * e[j + 1]), pack_bf16(dsn * e[j + 2], dsn * e[j + 3]),
                                                pack_bf16(dsn * e[j + 4], dsn * e[j + 5]), pack_bf16(dsn * e[j + 6], dsn * e[j + 7])));
                        st_shared_v4(sw128_chunk(a3, row, 4 * half + q),
                                     make_uint4(pack_bf16(pg * dy[j], pg * dy[j + 1]), pack_bf16(pg * dy[j + 2], pg * dy[j + 3]),
                                                pack_bf16(pg * dy[j + 4], pg * dy[j + 5]), pack_bf16(pg * dy[j + 6], pg * dy[j + 7])));
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(A_FULL0 + (c & 1)));
                }
                if (inrow) {
                    const size_t w = (bh * p.C + c) * p.L + tok;
                    if (half == 0) p.pbuf[w] = pc; else p.dsbuf[w] = ds;
                }
            }
            // ---- the tile's outputs --------------------------------------
            if (ok) ok = mbar_wait_warp(bar(D_FULL), 0, wc, 8);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    float a[32], b[32];
                    const uint32_t col = (uint32_t)(half * 64 + part * 32);
                    tmem_ld_32x32b_x32(t_lane + kColDQ + col, a);
                    tmem_ld_32x32b_x32(t_lane + kColDC + col, b);
                    tmem_ld_wait();
                    if (inrow) {
                        float4* q4 = reinterpret_cast<float4*>(p.dQ + orow * kN + col);
                        float4* c4 = reinterpret_cast<float4*>(p.dCh + orow * kN + col);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            q4[j] = make_float4(a[4 * j], a[4 * j + 1], a[4 * j + 2], a[4 * j + 3]);
                            c4[j] = make_float4(b[4 * j], b[4 * j + 1], b[4 * j + 2], b[4 * j + 3]);
                        }
                    }
                }
                if (inrow) {
                    float4* e4 = reinterpret_cast<float4*>(p.dE + orow * kP + col0);
#pragma unroll
                    for (int j = 0; j < 8; ++j) e4[j] = make_float4(de[4 * j], de[4 * j + 1], de[4 * j + 2], de[4 * j + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ===========================================================================
// memory side
// ===========================================================================
namespace ms {
// One CTA per pair of consecutive memories (c0 = 2m, c1 = 2m + 1) of one
// (b, h): the query tiles of chunk c0 + 1 feed c0 alone, every later tile
// feeds both, so each E and dy row a builder loads serves two memories and
// each Q and C tile two products.
constexpr uint32_t kOffQ = 0;                   // 2 panels (one buffer)
constexpr uint32_t kOffC = 2 * kPanel;          // 2 panels (one buffer)
constexpr uint32_t kOffOps = 4 * kPanel;        // 2 buffers x [E0, D0, E1, D1] operand rows
constexpr uint32_t kOpsBuf = 4 * kPanel;
constexpr uint32_t kOffBar = kOffOps + 2 * kOpsBuf;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
constexpr int kBuilders = 4;
constexpr int kThreads = 64 + 32 * kBuilders;
enum Bar { QC_FULL = 0, QC_EMPTY = 1, OP_FULL0 = 2, OP_EMPTY0 = 4, D_FULL = 6, NUM_BARS = 7 };
static_assert(NUM_BARS * 8 + 8 <= 256 && kSmemBytes <= 232448, "shared memory layout");
}  // namespace ms

__global__ void __launch_bounds__(ms::kThreads, 1) sma_bwd_dh_tc(const __grid_constant__ SmaBwdTcParams p) {
    using namespace ms;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffBar + NUM_BARS * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // memory pair m of (b, h), in order of increasing m (most attending tokens first)
    const int per_m = p.B * p.H;
    const int m = blockIdx.x / per_m, bhi = blockIdx.x % per_m;
    const int b = bhi / p.H, h = bhi % p.H;
    const size_t bh = (size_t)b * p.H + h;
    const int c0 = 2 * m, c1 = 2 * m + 1;
    // query tiles of chunks c0+1 .. C-1 that start before L; tiles j >= tpc also attend c1
    int ntiles = (p.C - 1 - c0) * p.tpc;
    while (ntiles > 0 && (c0 + 1 + (ntiles - 1) / p.tpc) * p.S + ((ntiles - 1) % p.tpc) * kBQ >= p.L) --ntiles;
    auto tile_t0 = [&](int j) { return (c0 + 1 + j / p.tpc) * p.S + (j % p.tpc) * kBQ; };
    auto both = [&](int j) { return j >= p.tpc; };
    const bool has_c1 = c1 < p.C;
    const bool c1_tiles = has_c1 && ntiles > p.tpc;

    if (threadIdx.x == 0) {
        mbar_init(bar(QC_FULL), 1);
        mbar_init(bar(QC_EMPTY), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(OP_FULL0 + i), kBuilders);
            mbar_init(bar(OP_EMPTY0 + i), 1);
        }
        mbar_init(bar(D_FULL), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tmap_q);
        tma_prefetch_desc(&p.tmap_c);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 128);   // ddH[c0] in columns 0-63, ddH[c1] in 64-127
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const WaitCtx wc{abort_flag, p.status, 5};

    if (warp == 0) {
        bool ok = true;
        for (int j = 0; j < ntiles && ok; ++j) {
            const int t0 = tile_t0(j);
            if (!(ok = mbar_wait_warp(bar(QC_EMPTY), ((uint32_t)j & 1u) ^ 1u, wc, 1))) break;
            if (lane == 0) {
                mbar_expect_tx(bar(QC_FULL), 4 * kPanel);
                tma_load_4d(sbase + kOffQ, &p.tmap_q, bar(QC_FULL), 0, h, t0, b);
                tma_load_4d(sbase + kOffQ + kPanel, &p.tmap_q, bar(QC_FULL), 64, h, t0, b);
                tma_load_4d(sbase + kOffC, &p.tmap_c, bar(QC_FULL), 0, h / p.HG, t0, b);
                tma_load_4d(sbase + kOffC + kPanel, &p.tmap_c, bar(QC_FULL), 64, h / p.HG, t0, b);
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        bool ok = true;
        const uint32_t idesc = idesc_bf16_f32(kN, kP, true, true);   // A = Q^T, C^T (MN-major), B MN-major
        for (int j = 0; j < ntiles && ok; ++j) {
            const int buf = j & 1;
            if (!(ok = mbar_wait_warp(bar(QC_FULL), (uint32_t)j & 1u, wc, 2))) break;
            if (!(ok = mbar_wait_warp(bar(OP_FULL0 + buf), (uint32_t)(j >> 1) & 1u, wc, 3))) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t ops = sbase + kOffOps + (uint32_t)buf * kOpsBuf;
                const int nmem = both(j) ? 2 : 1;
                for (int mm = 0; mm < nmem; ++mm) {
                    const uint32_t d = tmem + (uint32_t)(64 * mm);
                    const bool first = mm == 0 ? j == 0 : j == p.tpc;
                    const uint32_t be = ops + (uint32_t)(2 * mm) * kPanel, bdo = be + kPanel;
#pragma unroll 1
                    for (int kk = 0; kk < kBQ / 16; ++kk) {
                        const uint32_t ko = (uint32_t)kk * 2048;   // 16 token rows
                        mma_f16_ss(d, smem_desc_sw128(sbase + kOffQ + ko, kPanel, 1024),
                                   smem_desc_sw128(be + ko, kPanel, 1024), idesc, (!first || kk > 0) ? 1u : 0u);
                        mma_f16_ss(d, smem_desc_sw128(sbase + kOffC + ko, kPanel, 1024),
                                   smem_desc_sw128(bdo + ko, kPanel, 1024), idesc, 1u);
                    }
                }
                mma_commit(bar(QC_EMPTY));
                mma_commit(bar(OP_EMPTY0 + buf));
                if (j == ntiles - 1) mma_commit(bar(D_FULL));
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------- operand builders
        const int quad = warp & 3;
        const int r = quad * 32 + lane;                 // token row of a tile / state row n at the end
        const float inv_sqrt_n = rsqrtf((float)kN);
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            const int buf = j & 1, tok = tile_t0(j) + r;
            if (ok) ok = mbar_wait_warp(bar(OP_EMPTY0 + buf), ((uint32_t)(j >> 1) & 1u) ^ 1u, wc, 4);
            if (!ok) continue;
            const uint32_t ops = sbase + kOffOps + (uint32_t)buf * kOpsBuf;
            const int nmem = both(j) ? 2 : 1;
            if (tok < p.L) {
                float dsn[2], pg[2];
#pragma unroll
                for (int mm = 0; mm < 2; ++mm) {
                    if (mm < nmem) {
                        const size_t w = (bh * p.C + c0 + mm) * p.L + tok;
                        dsn[mm] = __ldg(p.dsbuf + w) * inv_sqrt_n;
                        pg[mm] = __ldg(p.pbuf + w) * p.g;
                    } else {
                        dsn[mm] = pg[mm] = 0.f;
                    }
                }
                const size_t orow = ((size_t)b * p.L + tok) * p.H + h;
                const uint4* es = reinterpret_cast<const uint4*>(p.E + orow * kP);
                const float4* dys = reinterpret_cast<const float4*>(p.dy + orow * kP);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float ev[8];
                    widen8(__ldg(es + q), ev);
                    const float4 y0 = __ldg(dys + 2 * q), y1 = __ldg(dys + 2 * q + 1);
#pragma unroll
                    for (int mm = 0; mm < 2; ++mm) {
                        if (mm < nmem) {
                            const float a = dsn[mm], g = pg[mm];
                            st_shared_v4(sw128_chunk(ops + (uint32_t)(2 * mm) * kPanel, r, q),
                                         make_uint4(pack_bf16(a * ev[0], a * ev[1]), pack_bf16(a * ev[2], a * ev[3]),
                                                    pack_bf16(a * ev[4], a * ev[5]), pack_bf16(a * ev[6], a * ev[7])));
                            st_shared_v4(sw128_chunk(ops + (uint32_t)(2 * mm + 1) * kPanel, r, q),
                                         make_uint4(pack_bf16(g * y0.x, g * y0.y), pack_bf16(g * y0.z, g * y0.w),
                                                    pack_bf16(g * y1.x, g * y1.y), pack_bf16(g * y1.z, g * y1.w)));
                        }
                    }
                }
            } else {
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int q = 0; q < 8; ++q)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (k < 2 * nmem) st_shared_v4(sw128_chunk(ops + (uint32_t)k * kPanel, r, q), z);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(OP_FULL0 + buf));
        }
        // ddH[c0] and ddH[c1]: row r = state row n
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        if (ntiles > 0 && ok) ok = mbar_wait_warp(bar(D_FULL), 0, wc, 5);
        if (ok) tc_fence_after();
#pragma unroll 1
        for (int mm = 0; mm < 2; ++mm) {
            if (mm == 1 && !has_c1) break;
            float* out = p.ddH + ((bh * p.C + c0 + mm) * kN + r) * (size_t)kP;
            const bool any = mm == 0 ? ntiles > 0 : c1_tiles;
            if (!any) {
                const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int q = 0; q < 16; ++q) reinterpret_cast<float4*>(out)[q] = z;
            } else if (ok) {
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    float a[32];
                    tmem_ld_32x32b_x32(t_lane + (uint32_t)(64 * mm + 32 * part), a);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        reinterpret_cast<float4*>(out + part * 32)[q] =
                            make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

}  // namespace

bool sma_bwd_tc_applicable(int N, int P, int S, dart_dtype dt) {
    return dt == DART_BF16 && N == kN && P == kP && S % kBQ == 0 && S <= 65536;
}

int sma_bwd_tc_tiles(int B, int L, int H, int S) {
    const int C = (L + S - 1) / S;
    return B * H * C * (S / kBQ);
}

cudaError_t launch_sma_bwd_tc(const SmaBwdArgs& a, cudaStream_t st) {
    SmaBwdTcParams p;
    memset(&p, 0, sizeof(p));
    const int C = (a.L + a.S - 1) / a.S;
    {
        const uint64_t dims[4] = {(uint64_t)kN, (uint64_t)a.H, (uint64_t)a.L, (uint64_t)a.B};
        const uint64_t strides[3] = {(uint64_t)kN * 2, (uint64_t)a.H * kN * 2, (uint64_t)a.L * a.H * kN * 2};
        const uint32_t box[4] = {64, 1, kBQ, 1};
        if (!encode_tile_map_bf16(&p.tmap_q, 4, a.Q, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[4] = {(uint64_t)kN, (uint64_t)a.G, (uint64_t)a.L, (uint64_t)a.B};
        const uint64_t strides[3] = {(uint64_t)kN * 2, (uint64_t)a.G * kN * 2, (uint64_t)a.L * a.G * kN * 2};
        const uint32_t box[4] = {64, 1, kBQ, 1};
        if (!encode_tile_map_bf16(&p.tmap_c, 4, a.Cm, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[2] = {(uint64_t)kP, (uint64_t)a.B * a.H * C * kN};
        const uint64_t strides[1] = {(uint64_t)kP * 2};
        const uint32_t box[2] = {kP, kN};
        if (!encode_tile_map_bf16(&p.tmap_h, 2, a.dH, dims, strides, box)) return cudaErrorInvalidValue;
    }
    p.E = static_cast<const __nv_bfloat16*>(a.E);
    p.dy = a.dy;
    p.g = a.g;
    p.B = a.B; p.L = a.L; p.H = a.H; p.S = a.S; p.C = C;
    p.HG = a.H / a.G;
    p.tpc = a.S / kBQ;
    p.dQ = a.dQ; p.dE = a.dE; p.dCh = a.dCh; p.ddH = a.ddH;
    p.pbuf = a.pbuf; p.dsbuf = a.dsbuf; p.gpart = a.gpart;
    p.status = a.status;
    cudaError_t e;
    {
        auto k = sma_bwd_q_tc;
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qs::kSmemBytes)) != cudaSuccess)
            return e;
        k<<<sma_bwd_tc_tiles(a.B, a.L, a.H, a.S), qs::kThreads, qs::kSmemBytes, st>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        auto k = sma_bwd_dh_tc;
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ms::kSmemBytes)) != cudaSuccess)
            return e;
        k<<<a.B * a.H * ((C + 1) / 2), ms::kThreads, ms::kSmemBytes, st>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    count_launches(2);
    return cudaSuccess;
}

}  // namespace dart
