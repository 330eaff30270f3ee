// ssd_scan_bwd_tc.cu -- the intra-chunk part of the scan backward on the
// 5th-generation tensor cores, in the quadratic (SSD) form.
//
// Notation of ssd_scan_bwd.cu: chunk c with tokens s0..e, Acum_t the
// in-chunk prefix of dt A_h, Ae = Acum_e, R = Gin[c] + gD[c] (the adjoint
// entering the chunk from later chunks plus the memory gradient), h_in the
// state entering the chunk, f_t = exp(Ae - Acum_t).  Unrolling the token
// adjoints inside the chunk gives, for every token t,
//   dx_t / dt_t = sum_{s>=t} exp(Acum_s - Acum_t) (B_t . C_s) dy_s + f_t R^T B_t
//   dB_t / dt_t = sum_{s>=t} exp(Acum_s - Acum_t) (x_t . dy_s) C_s + f_t R x_t
//   dC_t        = sum_{r<=t} exp(Acum_t - Acum_r) dt_r (dy_t . x_r) B_r + exp(Acum_t) h_in dy_t
// (dB, dC per head), and the scalars the decay gradient needs:
//   q1_t = x_t . (dx_t / dt_t),  u_t = x_t . (R^T B_t),  v_t = dy_t . (h_in^T C_t),
//   colsum_t = sum_{s>t} W_{s,t},  rowsum_t = sum_{r<t} W_{t,r},
//   W_{s,r} = exp(Acum_s - Acum_r) dt_r (C_s . B_r)(dy_s . x_r).
// Rect_t = sum_{r<t<=s} W_{s,r} is a small difference of the running row and
// column sums, so both sums are taken from the same W values (each pair once,
// in the upper blocks): a W rounded two different ways cancels badly there.
// scan_bwd_scalars (ssd_scan_bwd.cu) turns them into ddt and dA by three
// recursions over the chunk's tokens, each run as a warp scan.
//
// One CTA per (b, h, c, 128-token row block i) computes those for its rows:
//   steps 0-2    B_i R and C_i h_in (for u, v); dx += (f B_i) R,
//                dB += (f x_i) R^T, dC += (exp(Acum) dy_i) h_in^T;
//   upper blocks j >= i:   G = B_i C_j^T -> M_x = mask o decay o G (bf16)
//                dx += M_x dy_j;  G = x_i dy_j^T -> W = dt M_x o G: its sums over
//                s (per thread) and over t (warp transpose-reduce, then the four
//                warps in order); M_b -> dB += M_b C_j;
//   lower blocks j <= i:   G = dy_i x_j^T -> M_c -> dC += M_c B_j;
// then dx, dB, dC leave TMEM and the scalars go to the workspace.  The
// steps run one after another (an MMA step, then the row threads).
// TMEM: dx (64 columns), dB (128), dC (128), one 128-column scratch block.
// Operands are bf16: B, C, x as given, dy, R, h_in and the M tiles rounded
// once (2^-9 relative); products accumulate in fp32.
#include <cuda_bf16.h>
#include <string.h>

#include "dart_backward.cuh"
#include "sm100.cuh"
#include "tensor_map.h"

namespace dart {
namespace {

using namespace sm100;

constexpr int kN = 128, kP = 64, kRB = 128;   // compiled shape; tokens per row block
constexpr uint32_t kPanel = 128 * 64 * 2;     // 128 rows x 64 bf16, one 128-byte swizzle panel
constexpr uint32_t kOffBI = 0;                // B rows of block i (2 panels)
constexpr uint32_t kOffCI = 2 * kPanel;       // C rows of block i (2 panels)
constexpr uint32_t kOffXI = 4 * kPanel;       // x rows of block i
constexpr uint32_t kOffDI = 5 * kPanel;       // dy rows of block i (bf16)
constexpr uint32_t kOffR = 6 * kPanel;        // R [n][p]
constexpr uint32_t kOffH = 7 * kPanel;        // h_in [n][p]
constexpr uint32_t kOffO = 8 * kPanel;        // the other block: C_1 and dy_1 (block 0) or B_0 and x_0 (block 1)
constexpr uint32_t kOffOp = 11 * kPanel;      // operand rows built by the threads (2 panels)
constexpr uint32_t kOffF = 13 * kPanel;       // acum2[256], dtv[256], red[16], colred[4][128], xch[2][2][128] float2
constexpr uint32_t kOffBar = kOffF + 2 * 256 * 4 + 64 + 4 * 128 * 4 + 2 * 2 * 128 * 8;
constexpr uint32_t kSmemBytes = kOffBar + 64 + 1024;
constexpr int kThreads = 64 + 256;   // TMA, MMA, two warps per TMEM lane quadrant
constexpr uint32_t kColDX = 0, kColDB = 64, kColDC = 192, kColG = 320;
enum Bar { LD = 0, PREP = 1, MMA_DONE = 2, OP_READY = 3, NUM_BARS = 4 };
static_assert(kSmemBytes <= 232448 && NUM_BARS * 8 + 8 <= 64, "shared memory layout");

struct ScanBwdTcParams {
    CUtensorMap tmap_b, tmap_c;   // (N, G, L, B), box (64, 1, 128, 1)
    CUtensorMap tmap_x;           // (P, H, L, B), box (64, 1, 128, 1)
    const float* dt; const float* A; const float* dy;
    float* gin;    // the chunk adjoints: dS written by scan_bwd_dS_tc, Gin read by scan_bwd_quad_tc
    const float* ddH; const float* states; const float* init;
    float* dx; float* dBh; float* dCh;
    float* scal;   // [6][B,H,C,S]: u, v, q1, colsum, rowsum parts of row blocks 0 and 1
    float* asum;   // [B,H,C] chunk decay sums (written by scan_bwd_dS_tc)
    float* c0;     // [B,H,C]: sum(Gin o h_in)
    int B, L, H, S, C, HG, R;
    int* status;
};

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
__device__ __forceinline__ uint4 pack8(const float* f) {
    return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
}
// Byte address of 16-byte chunk q (8 bf16) of row r of a 128-byte-swizzled panel.
__device__ __forceinline__ uint32_t chunk_addr(uint32_t panel, int r, int q) {
    return panel + (uint32_t)r * 128u + ((uint32_t)(q ^ (r & 7)) << 4);
}
__device__ __forceinline__ void st_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ uint4 ld_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
// Row r of a bf16 operand of 64 * np columns (np panels) as fp32, 8 at a time.
__device__ __forceinline__ void ld_row8(uint32_t base, int r, int q, float* f) {
    widen8(ld_v4(chunk_addr(base + (uint32_t)(q >> 3) * kPanel, r, q & 7)), f);
}
__device__ __forceinline__ void st_row8(uint32_t base, int r, int q, const float* f) {
    st_v4(chunk_addr(base + (uint32_t)(q >> 3) * kPanel, r, q & 7), pack8(f));
}
// fp32 row (64 values) from global into a bf16 panel row, zeros if !valid.
__device__ __forceinline__ void row_to_bf16(uint32_t panel, int r, const float* src, bool valid) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float f[8];
        if (valid) {
            const float4 a = __ldg(reinterpret_cast<const float4*>(src) + 2 * q);
            const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 2 * q + 1);
            f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) f[k] = 0.f;
        }
        st_v4(chunk_addr(panel, r, q), pack8(f));
    }
}

__global__ void __launch_bounds__(kThreads, 1) scan_bwd_quad_tc(const __grid_constant__ ScanBwdTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    float* acum2 = reinterpret_cast<float*>(smem + kOffF);   // log2(e) Acum over the chunk
    float* dtv = acum2 + 256;
    float* red = dtv + 256;                                  // [8] c0 partials
    float* colred = red + 16;                                // [4 warps][128 columns] W sums
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffBar + NUM_BARS * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    auto bar = [&](int i) -> uint32_t { return sb + kOffBar + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x % p.R;
    const int c = (blockIdx.x / p.R) % p.C;
    const int bh = blockIdx.x / (p.R * p.C);
    const int b = bh / p.H, h = bh % p.H, grp = h / p.HG;
    const size_t bhc = (size_t)bh * p.C + c;
    const int s0 = c * p.S, n_chunk = min(p.L, s0 + p.S) - s0;
    const int t0 = s0 + i * kRB;                              // first token of the row block
    const bool other = p.R == 2;                              // a second block of the chunk exists

    if (threadIdx.x == 0) {
        mbar_init(bar(LD), 1);
        mbar_init(bar(PREP), 8);
        mbar_init(bar(MMA_DONE), 1);
        mbar_init(bar(OP_READY), 8);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const WaitCtx wc{abort_flag, p.status, 6};
    // steps: 0-2, then 3 per upper block (j = i .. R-1) and 2 per lower block (j = 0 .. i)
    const int nsteps = 3 + 3 * (p.R - i) + 2 * (i + 1);

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA
        if (lane == 0) {
            tma_prefetch_desc(&p.tmap_b);
            tma_prefetch_desc(&p.tmap_c);
            tma_prefetch_desc(&p.tmap_x);
            uint32_t bytes = 5 * kPanel;
            if (other) bytes += i == 0 ? 2 * kPanel : 3 * kPanel;
            mbar_expect_tx(bar(LD), bytes);
            tma_load_4d(sb + kOffBI, &p.tmap_b, bar(LD), 0, grp, t0, b);
            tma_load_4d(sb + kOffBI + kPanel, &p.tmap_b, bar(LD), 64, grp, t0, b);
            tma_load_4d(sb + kOffCI, &p.tmap_c, bar(LD), 0, grp, t0, b);
            tma_load_4d(sb + kOffCI + kPanel, &p.tmap_c, bar(LD), 64, grp, t0, b);
            tma_load_4d(sb + kOffXI, &p.tmap_x, bar(LD), 0, h, t0, b);
            if (other && i == 0) {          // C of block 1 (its dy is converted by the threads)
                tma_load_4d(sb + kOffO, &p.tmap_c, bar(LD), 0, grp, s0 + kRB, b);
                tma_load_4d(sb + kOffO + kPanel, &p.tmap_c, bar(LD), 64, grp, s0 + kRB, b);
            } else if (other) {             // B and x of block 0
                tma_load_4d(sb + kOffO, &p.tmap_b, bar(LD), 0, grp, s0, b);
                tma_load_4d(sb + kOffO + kPanel, &p.tmap_b, bar(LD), 64, grp, s0, b);
                tma_load_4d(sb + kOffO + 2 * kPanel, &p.tmap_x, bar(LD), 0, h, s0, b);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        bool ok = mbar_wait_warp(bar(LD), 0, wc, 1);
        if (ok) ok = mbar_wait_warp(bar(PREP), 0, wc, 2);
        const uint32_t id_n64_bmn = idesc_bf16_f32(128, 64, false, true);
        const uint32_t id_n128_bk = idesc_bf16_f32(128, 128, false, false);
        const uint32_t id_n128_bmn = idesc_bf16_f32(128, 128, false, true);
        // D (+)= A x B with A K-major (ka panels of K), B K-major or MN-major
        auto mma_kk = [&](uint32_t d, uint32_t a, uint32_t bop, bool b_mn, uint32_t b_lbo, int ksteps, uint32_t idesc,
                          bool acc0) {
#pragma unroll 1
            for (int kk = 0; kk < ksteps; ++kk) {
                const uint64_t ad = smem_desc_sw128(a + (uint32_t)(kk >> 2) * kPanel + (uint32_t)(kk & 3) * 32, 16, 1024);
                const uint64_t bd = b_mn ? smem_desc_sw128(bop + (uint32_t)kk * 2048, b_lbo, 1024)
                                         : smem_desc_sw128(bop + (uint32_t)(kk >> 2) * kPanel + (uint32_t)(kk & 3) * 32, 16, 1024);
                mma_f16_ss(d, ad, bd, idesc, (acc0 || kk > 0) ? 1u : 0u);
            }
        };
        for (int r = 0; r < nsteps && ok; ++r) {
            if (r > 0 && !(ok = mbar_wait_warp(bar(OP_READY), (uint32_t)(r - 1) & 1u, wc, 3))) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t op = sb + kOffOp;
                if (r == 0) {            // B_i R (u) and C_i h_in (v) into the scratch block
                    mma_kk(tmem + kColG, sb + kOffBI, sb + kOffR, true, kPanel, 8, id_n64_bmn, false);
                    mma_kk(tmem + kColG + 64, sb + kOffCI, sb + kOffH, true, kPanel, 8, id_n64_bmn, false);
                } else if (r == 1) {     // dx = (f B_i) R
                    mma_kk(tmem + kColDX, op, sb + kOffR, true, kPanel, 8, id_n64_bmn, false);
                } else if (r == 2) {     // dB = (f x_i) R^T, dC = (exp(Acum) dy_i) h_in^T
                    mma_kk(tmem + kColDB, op, sb + kOffR, false, 16, 4, id_n128_bk, false);
                    mma_kk(tmem + kColDC, op + kPanel, sb + kOffH, false, 16, 4, id_n128_bk, false);
                } else {
                    const int q = r - 3, nup = 3 * (p.R - i);
                    if (q < nup) {       // upper block j
                        const int j = i + q / 3, step = q % 3;
                        const uint32_t cj = j == i ? sb + kOffCI : sb + kOffO;
                        const uint32_t dyj = j == i ? sb + kOffDI : sb + kOffO + 2 * kPanel;
                        if (step == 0) {
                            mma_kk(tmem + kColG, sb + kOffBI, cj, false, 16, 8, id_n128_bk, false);       // B_i C_j^T
                        } else if (step == 1) {
                            mma_kk(tmem + kColDX, op, dyj, true, kPanel, 8, id_n64_bmn, true);           // dx += M_x dy_j
                            mma_kk(tmem + kColG, sb + kOffXI, dyj, false, 16, 4, id_n128_bk, false);     // x_i dy_j^T
                        } else {
                            mma_kk(tmem + kColDB, op, cj, true, kPanel, 8, id_n128_bmn, true);           // dB += M_b C_j
                        }
                    } else {             // lower block j
                        const int j = (q - nup) / 2, step = (q - nup) % 2;
                        const uint32_t bj = j == i ? sb + kOffBI : sb + kOffO;
                        const uint32_t xj = j == i ? sb + kOffXI : sb + kOffO + 2 * kPanel;
                        if (step == 0) {
                            mma_kk(tmem + kColG, sb + kOffDI, xj, false, 16, 4, id_n128_bk, false);      // dy_i x_j^T
                        } else {
                            mma_kk(tmem + kColDC, op, bj, true, kPanel, 8, id_n128_bmn, true);           // dC += M_c B_j
                        }
                    }
                }
                mma_commit(bar(MMA_DONE));
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------- the rows
        // Two warps per TMEM lane quadrant: warp half h owns the value columns
        // [32h, 32h+32), the state columns [64h, 64h+64) and the token columns
        // [64h, 64h+64) of every 128-column block; the row sums of the two
        // halves are exchanged in shared memory.
        const int quad = warp & 3, half = (warp - 2) >> 2;
        const int row = quad * 32 + lane;
        const int tl = i * kRB + row;            // token index within the chunk
        const bool valid = tl < n_chunk;
        const size_t tok = (size_t)b * p.L + s0 + tl;
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        const float Ah = p.A[h];
        float2* xch = reinterpret_cast<float2*>(colred + 4 * 128);   // [2 parity][2 half][128 rows]
        int xi = 0;
        // (a, b) of this row plus the other half's
        auto exchange = [&](float a, float bb) -> float2 {
            xch[((xi & 1) * 2 + half) * 128 + row] = make_float2(a, bb);
            named_bar_sync(2 + quad, 64);
            const float2 o = xch[((xi & 1) * 2 + (1 - half)) * 128 + row];
            ++xi;
            return make_float2(a + o.x, bb + o.y);
        };
        // the chunk's log2 decay prefix (warp 2), then everyone
        if (warp == 2) {
            const int per = (p.S + 31) / 32, a0 = lane * per;
            float run = 0.f;
            for (int k = 0; k < per && a0 + k < p.S; ++k) {
                const int t = a0 + k;
                const float d = t < n_chunk ? p.dt[((size_t)b * p.L + s0 + t) * p.H + h] : 0.f;
                dtv[t] = d;
                run += d * Ah * kLog2e;
                acum2[t] = run;
            }
            float off = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, off, o);
                if (lane >= o) off += v;
            }
            off -= run;
            for (int k = 0; k < per && a0 + k < p.S; ++k) acum2[a0 + k] += off;
        }
        // 8 floats of a 256-byte-aligned row at 8 q
        auto ld8 = [](const float* src, int q, float* f) {
            const float4 a = __ldg(reinterpret_cast<const float4*>(src) + 2 * q);
            const float4 d = __ldg(reinterpret_cast<const float4*>(src) + 2 * q + 1);
            f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = d.x; f[5] = d.y; f[6] = d.z; f[7] = d.w;
        };
        // this half's columns of dy (block i, and block 1 for block 0), R and h_in as bf16; c0
        {
            auto dy_half = [&](uint32_t panel, int r, const float* src, bool ok_row) {
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int q = 4 * half + qq;
                    float f[8];
                    if (ok_row) ld8(src, q, f);
                    else {
#pragma unroll
                        for (int k = 0; k < 8; ++k) f[k] = 0.f;
                    }
                    st_v4(chunk_addr(panel, r, q), pack8(f));
                }
            };
            dy_half(sb + kOffDI, row, p.dy + (tok * p.H + h) * kP, valid);
            if (other && i == 0) {
                const int tl1 = kRB + row;
                dy_half(sb + kOffO + 2 * kPanel, row, p.dy + (((size_t)b * p.L + s0 + tl1) * p.H + h) * kP,
                        tl1 < n_chunk);
            }
            const int n = row;
            const float* gi = p.gin + (bhc * kN + n) * kP;
            const float* gd = p.ddH ? p.ddH + (bhc * kN + n) * kP : nullptr;
            const float* hi = c > 0 ? p.states + (((size_t)bh * p.C + (c - 1)) * kN + n) * kP
                                    : (p.init ? p.init + ((size_t)bh * kN + n) * kP : nullptr);
            float c0p = 0.f;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const int q = 4 * half + qq;
                float g8[8], d8[8], h8[8];
                ld8(gi, q, g8);
                if (gd) ld8(gd, q, d8);
                if (hi) ld8(hi, q, h8);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (!hi) h8[k] = 0.f;
                    c0p = fmaf(g8[k], h8[k], c0p);
                    g8[k] += gd ? d8[k] : 0.f;   // R = Gin + gD
                }
                st_v4(chunk_addr(sb + kOffR, n, q), pack8(g8));
                st_v4(chunk_addr(sb + kOffH, n, q), pack8(h8));
            }
            c0p = warp_sum(c0p);
            if (lane == 0) red[warp - 2] = c0p;
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 256);                  // acum2, dtv and red visible to all row threads
        if (threadIdx.x == 64 && i == 0)
            p.c0[bhc] = ((red[0] + red[1]) + (red[2] + red[3])) + ((red[4] + red[5]) + (red[6] + red[7]));
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(PREP));
        bool ok = mbar_wait_warp(bar(LD), 0, wc, 4);   // the TMA rows are read below
        const float a2t = acum2[tl < p.S ? tl : p.S - 1];
        const float a2e = acum2[p.S - 1];
        const float f_t = exp2f(a2e - a2t);            // exp(Ae - Acum_t)
        const float e_t = exp2f(a2t);                  // exp(Acum_t)
        const float dtt = valid ? dtv[tl] : 0.f;
        float colsum = 0.f;
        int rd = 0;                                    // MMA steps completed
        auto wait_step = [&]() {
            if (ok) ok = mbar_wait_warp(bar(MMA_DONE), (uint32_t)rd & 1u, wc, 5);
            ++rd;
            tc_fence_after();
        };
        auto done_step = [&]() {
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(OP_READY));
        };
        const uint32_t op = sb + kOffOp;
        // ---- step 0: u, v; operand f B_i -----------------------------------
        wait_step();
        {
            float rb[32], hc[32];
            if (ok) {
                tmem_ld_32x32b_x32(t_lane + kColG + (uint32_t)(32 * half), rb);
                tmem_ld_32x32b_x32(t_lane + kColG + 64 + (uint32_t)(32 * half), hc);
                tmem_ld_wait();
            }
            float u = 0.f, v = 0.f;
            const float* dyr = p.dy + (tok * p.H + h) * kP;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const int q = 4 * half + qq;
                float xv[8], dv[8];
                ld_row8(sb + kOffXI, row, q, xv);
                if (valid) ld8(dyr, q, dv);
                else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) dv[k] = 0.f;
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    u = fmaf(xv[k], rb[8 * qq + k], u);
                    v = fmaf(dv[k], hc[8 * qq + k], v);
                }
            }
            const float2 uv = exchange(u, v);
            if (valid && half == 0) {
                const size_t o = bhc * p.S + tl, plane = (size_t)p.B * p.H * p.C * p.S;
                p.scal[o] = uv.x;
                p.scal[plane + o] = uv.y;
            }
#pragma unroll
            for (int qq = 0; qq < 8; ++qq) {
                const int q = 8 * half + qq;
                float bv[8];
                ld_row8(sb + kOffBI, row, q, bv);
#pragma unroll
                for (int k = 0; k < 8; ++k) bv[k] *= f_t;
                st_row8(op, row, q, bv);
            }
        }
        done_step();
        // ---- step 1: operands f x_i and exp(Acum) dy_i -----------------------
        wait_step();
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const int q = 4 * half + qq;
            float xv[8], dv[8];
            ld_row8(sb + kOffXI, row, q, xv);
            ld_row8(sb + kOffDI, row, q, dv);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                xv[k] *= f_t;
                dv[k] *= e_t;
            }
            st_row8(op, row, q, xv);
            st_row8(op + kPanel, row, q, dv);
        }
        done_step();
        // ---- step 2: nothing to build --------------------------------------
        wait_step();
        done_step();
        // ---- upper blocks -----------------------------------------------------
        for (int j = i; j < p.R; ++j) {
            // B_i C_j^T -> M_x
            wait_step();
#pragma unroll 1
            for (int pp = 0; pp < 2; ++pp) {
                const int part = 2 * half + pp;
                float g[32];
                if (ok) {
                    tmem_ld_32x32b_x32(t_lane + kColG + (uint32_t)(32 * part), g);
                    tmem_ld_wait();
                }
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const int sl = j * kRB + 32 * part + k;
                    g[k] = sl >= tl ? exp2f(acum2[sl] - a2t) * g[k] : 0.f;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) st_row8(op, row, 4 * part + q, g + 8 * q);
            }
            done_step();
            // x_i dy_j^T -> W = dt_t M_x o G (s > t) summed over s (colsum of t)
            // and over t (this block's part of rowsum of s); M_b
            wait_step();
#pragma unroll 1
            for (int pp = 0; pp < 2; ++pp) {
                const int part = 2 * half + pp;
                float g[32], mx[32], w[32];
                if (ok) {
                    tmem_ld_32x32b_x32(t_lane + kColG + (uint32_t)(32 * part), g);
                    tmem_ld_wait();
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) ld_row8(op, row, 4 * part + q, mx + 8 * q);
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const int sl = j * kRB + 32 * part + k;
                    w[k] = sl > tl ? dtt * mx[k] * g[k] : 0.f;
                    colsum += w[k];
                    g[k] = sl >= tl ? exp2f(acum2[sl] - a2t) * g[k] : 0.f;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) st_row8(op, row, 4 * part + q, g + 8 * q);
                // sums over the warp's 32 rows: after the halving steps lane l holds column l
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) {
                    const bool up = (lane & off) != 0;
#pragma unroll
                    for (int k = 0; k < off; ++k) {
                        const float send = up ? w[k] : w[k + off];
                        const float keep = up ? w[k + off] : w[k];
                        w[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                    }
                }
                colred[quad * 128 + 32 * part + lane] = w[0];
            }
            named_bar_sync(1, 256);
            if (half == 0) {   // column `row` of block j: the four quadrants' sums in order
                const float rs = (colred[row] + colred[128 + row]) + (colred[256 + row] + colred[384 + row]);
                const size_t plane = (size_t)p.B * p.H * p.C * p.S;
                p.scal[(size_t)(4 + i) * plane + bhc * p.S + j * kRB + row] = rs;
            }
            done_step();
            // dB += M_b C_j
            wait_step();
            done_step();
        }
        // ---- lower blocks -----------------------------------------------------
        for (int j = 0; j <= i; ++j) {
            // dy_i x_j^T -> M_c
            wait_step();
#pragma unroll 1
            for (int pp = 0; pp < 2; ++pp) {
                const int part = 2 * half + pp;
                float g[32];
                if (ok) {
                    tmem_ld_32x32b_x32(t_lane + kColG + (uint32_t)(32 * part), g);
                    tmem_ld_wait();
                }
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const int rl = j * kRB + 32 * part + k;
                    g[k] = rl <= tl ? exp2f(a2t - acum2[rl]) * dtv[rl] * g[k] : 0.f;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) st_row8(op, row, 4 * part + q, g + 8 * q);
            }
            done_step();
            // dC += M_c B_j
            wait_step();
            if (j < i) done_step();   // the last step hands nothing back
        }
        // ---- outputs -----------------------------------------------------------
        {
            float q1 = 0.f;
            if (ok) {
                float v[32], xv[32];
                tmem_ld_32x32b_x32(t_lane + kColDX + (uint32_t)(32 * half), v);
                tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < 4; ++q) ld_row8(sb + kOffXI, row, 4 * half + q, xv + 8 * q);
#pragma unroll
                for (int k = 0; k < 32; ++k) q1 = fmaf(xv[k], v[k], q1);
                if (valid) {
                    float4* d4 = reinterpret_cast<float4*>(p.dx + (tok * p.H + h) * kP + 32 * half);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        d4[k] = make_float4(dtt * v[4 * k], dtt * v[4 * k + 1], dtt * v[4 * k + 2], dtt * v[4 * k + 3]);
                }
#pragma unroll 1
                for (int pp = 0; pp < 2; ++pp) {
                    const int part = 2 * half + pp;
                    tmem_ld_32x32b_x32(t_lane + kColDB + (uint32_t)(32 * part), v);
                    tmem_ld_wait();
                    if (valid) {
                        float4* d4 = reinterpret_cast<float4*>(p.dBh + (tok * p.H + h) * kN + 32 * part);
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            d4[k] = make_float4(dtt * v[4 * k], dtt * v[4 * k + 1], dtt * v[4 * k + 2], dtt * v[4 * k + 3]);
                    }
                    tmem_ld_32x32b_x32(t_lane + kColDC + (uint32_t)(32 * part), v);
                    tmem_ld_wait();
                    if (valid) {
                        float4* d4 = reinterpret_cast<float4*>(p.dCh + (tok * p.H + h) * kN + 32 * part);
#pragma unroll
                        for (int k = 0; k < 8; ++k) d4[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                    }
                }
            }
            const float2 qc = exchange(q1, colsum);    // both halves take part, also after a failed wait
            if (ok && valid && half == 0) {
                const size_t o = bhc * p.S + tl, plane = (size_t)p.B * p.H * p.C * p.S;
                p.scal[2 * plane + o] = qc.x;
                p.scal[3 * plane + o] = qc.y;
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
// dS[c] = sum_s exp(Acum_s) C_s dy_s^T  (N x P) and the chunk's decay sum
// ===========================================================================
// One CTA per (b, h, c): C_T (S x N, TMA) is the MN-major A operand (M = N),
// the rows exp(Acum_s) dy_s are built by four warps as two bf16 MN-major B
// operands, the rounded value and the remainder (together ~16 bits of the
// fp32 value, so dS and the adjoints built from it keep fp32-like accuracy),
// and the product accumulates in TMEM over the S tokens.
constexpr uint32_t ds_kOffC = 0;                 // 2 n-panels x S rows (S * 256 B)
constexpr uint32_t ds_kOffHi = 4 * kPanel;       // S rows x 128 B
constexpr uint32_t ds_kOffLo = 6 * kPanel;
constexpr uint32_t ds_kOffF = 8 * kPanel;        // acum2[256]
constexpr uint32_t ds_kOffBar = ds_kOffF + 256 * 4;
constexpr uint32_t ds_kSmemBytes = ds_kOffBar + 64 + 1024;
enum DsBar { DS_LD = 0, DS_OPS = 1, DS_DONE = 2, ds_NUM_BARS = 3 };
static_assert(ds_kSmemBytes <= 232448, "shared memory layout");

constexpr int kThreadsDS = 64 + 128;   // TMA, MMA, four row warps

__global__ void __launch_bounds__(kThreadsDS, 1) scan_bwd_dS_tc(const __grid_constant__ ScanBwdTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    float* acum2 = reinterpret_cast<float*>(smem + ds_kOffF);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + ds_kOffBar + ds_NUM_BARS * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    auto bar = [&](int i) -> uint32_t { return sb + ds_kOffBar + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x % p.C, bh = blockIdx.x / p.C;
    const int b = bh / p.H, h = bh % p.H, grp = h / p.HG;
    const size_t bhc = (size_t)bh * p.C + c;
    const int s0 = c * p.S, n_chunk = min(p.L, s0 + p.S) - s0;
    const uint32_t rowblk = (uint32_t)kRB * 128u;    // 128 rows of one panel
    const uint32_t cpanel = (uint32_t)p.R * rowblk;  // one n-panel over all S rows

    if (threadIdx.x == 0) {
        mbar_init(bar(DS_LD), 1);
        mbar_init(bar(DS_OPS), 4);
        mbar_init(bar(DS_DONE), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const WaitCtx wc{abort_flag, p.status, 7};

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&p.tmap_c);
            mbar_expect_tx(bar(DS_LD), (uint32_t)p.R * 2u * kPanel);
            for (int r = 0; r < p.R; ++r)
                for (int nb = 0; nb < 2; ++nb)
                    tma_load_4d(sb + ds_kOffC + (uint32_t)nb * cpanel + (uint32_t)r * rowblk, &p.tmap_c, bar(DS_LD), 64 * nb,
                                grp, s0 + r * kRB, b);
        }
        __syncwarp();
    } else if (warp == 1) {
        bool ok = mbar_wait_warp(bar(DS_LD), 0, wc, 1);
        if (ok) ok = mbar_wait_warp(bar(DS_OPS), 0, wc, 2);
        tc_fence_after();
        if (ok && lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kN, kP, true, true);   // A = C_T^T (MN-major), B MN-major
            const int ksteps = p.S / 16;
            for (int kk = 0; kk < ksteps; ++kk) {
                const uint64_t ad = smem_desc_sw128(sb + ds_kOffC + (uint32_t)kk * 2048, cpanel, 1024);
                mma_f16_ss(tmem, ad, smem_desc_sw128(sb + ds_kOffHi + (uint32_t)kk * 2048, kPanel, 1024), idesc,
                           kk > 0 ? 1u : 0u);
                mma_f16_ss(tmem, ad, smem_desc_sw128(sb + ds_kOffLo + (uint32_t)kk * 2048, kPanel, 1024), idesc, 1u);
            }
            mma_commit(bar(DS_DONE));
        }
        __syncwarp();
    } else {
        const int quad = warp & 3, row = quad * 32 + lane;
        const float Ah = p.A[h];
        if (warp == 2) {   // the chunk's log2 decay prefix and its sum
            const int per = (p.S + 31) / 32, a0 = lane * per;
            float run = 0.f;
            for (int k = 0; k < per && a0 + k < p.S; ++k) {
                const int t = a0 + k;
                run += (t < n_chunk ? p.dt[((size_t)b * p.L + s0 + t) * p.H + h] : 0.f) * Ah * kLog2e;
                acum2[t] = run;
            }
            float off = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, off, o);
                if (lane >= o) off += v;
            }
            off -= run;
            for (int k = 0; k < per && a0 + k < p.S; ++k) acum2[a0 + k] += off;
            if (lane == 31) p.asum[bhc] = (off + run) * (1.f / kLog2e);   // Ae = sum of dt A over the chunk
        }
        named_bar_sync(1, 128);
        for (int r = 0; r < p.R; ++r) {
            const int t = r * kRB + row;
            const bool valid = t < n_chunk;
            const float w = valid ? exp2f(acum2[t]) : 0.f;
            const float* src = p.dy + (((size_t)b * p.L + s0 + t) * p.H + h) * kP;
            const uint32_t hi = sb + ds_kOffHi + (uint32_t)r * rowblk, lo = sb + ds_kOffLo + (uint32_t)r * rowblk;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float f[8], g[8];
                if (valid) {
                    const float4 a = __ldg(reinterpret_cast<const float4*>(src) + 2 * q);
                    const float4 d = __ldg(reinterpret_cast<const float4*>(src) + 2 * q + 1);
                    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = d.x; f[5] = d.y; f[6] = d.z; f[7] = d.w;
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) f[k] = 0.f;
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    f[k] *= w;
                    g[k] = f[k] - __bfloat162float(__float2bfloat16_rn(f[k]));
                }
                st_v4(chunk_addr(hi, row, q), pack8(f));
                st_v4(chunk_addr(lo, row, q), pack8(g));
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(DS_OPS));
        bool ok = mbar_wait_warp(bar(DS_DONE), 0, wc, 3);
        if (ok) {
            tc_fence_after();
            float v[32];
            float* dst = p.gin + (bhc * kN + row) * kP;   // TMEM lane = state row n
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(32 * part), v);
                tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    reinterpret_cast<float4*>(dst + 32 * part)[k] =
                        make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

bool make_params(const ScanBwdArgs& a, ScanBwdTcParams& p) {
    memset(&p, 0, sizeof(p));
    const int C = (a.L + a.S - 1) / a.S;
    {
        const uint64_t dims[4] = {(uint64_t)kN, (uint64_t)a.G, (uint64_t)a.L, (uint64_t)a.B};
        const uint64_t strides[3] = {(uint64_t)kN * 2, (uint64_t)a.G * kN * 2, (uint64_t)a.L * a.G * kN * 2};
        const uint32_t box[4] = {64, 1, kRB, 1};
        if (!encode_tile_map_bf16(&p.tmap_b, 4, a.Bm, dims, strides, box)) return false;
        if (!encode_tile_map_bf16(&p.tmap_c, 4, a.Cm, dims, strides, box)) return false;
    }
    {
        const uint64_t dims[4] = {(uint64_t)kP, (uint64_t)a.H, (uint64_t)a.L, (uint64_t)a.B};
        const uint64_t strides[3] = {(uint64_t)kP * 2, (uint64_t)a.H * kP * 2, (uint64_t)a.L * a.H * kP * 2};
        const uint32_t box[4] = {64, 1, kRB, 1};
        if (!encode_tile_map_bf16(&p.tmap_x, 4, a.x, dims, strides, box)) return false;
    }
    p.dt = a.dt; p.A = a.A; p.dy = a.dy;
    p.gin = a.gin; p.ddH = a.ddH; p.states = a.states; p.init = a.init;
    p.dx = a.dx; p.dBh = a.dBh; p.dCh = a.dCh;
    p.scal = a.rect; p.c0 = a.c0; p.asum = a.asum;
    p.B = a.B; p.L = a.L; p.H = a.H; p.S = a.S; p.C = C; p.HG = a.H / a.G; p.R = a.S / kRB;
    p.status = a.status;
    return true;
}

}  // namespace

bool scan_bwd_tc_applicable(int N, int P, int S, dart_dtype dt) {
    return dt == DART_BF16 && N == kN && P == kP && (S == 128 || S == 256);
}

cudaError_t launch_scan_bwd_dS_tc(const ScanBwdArgs& a, cudaStream_t st) {
    ScanBwdTcParams p;
    if (!make_params(a, p)) return cudaErrorInvalidValue;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(scan_bwd_dS_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ds_kSmemBytes)) !=
        cudaSuccess)
        return e;
    scan_bwd_dS_tc<<<a.B * a.H * p.C, kThreadsDS, ds_kSmemBytes, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_scan_bwd_quad_tc(const ScanBwdArgs& a, cudaStream_t st) {
    ScanBwdTcParams p;
    if (!make_params(a, p)) return cudaErrorInvalidValue;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(scan_bwd_quad_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes)) !=
        cudaSuccess)
        return e;
    scan_bwd_quad_tc<<<a.B * a.H * p.C * p.R, kThreads, kSmemBytes, st>>>(p);
    return cudaGetLastError();
}

}  // namespace dart
