// ssd_scan_tc.cu -- the SSD chunked scan with retained chunk memories on the
// 5th-generation tensor cores (bf16 inputs, N = 128, P = 64, S in {128, 256}).
//
// Mamba-2 SSD chunked scan as used by DART ("Transformers are SSMs" SSD view,
// Eq. (4); Pith review of DART, "What carries the argument" for the retained
// chunk contribution dH[c]), in four launches:
//
//  chunk_decay     per (b, h, c): the in-chunk prefix Acum of dt A, Asum[c]
//      and three per-token decay terms the other kernels bulk-copy.
//  chunk_state_tc  persistent, one CTA per SM over equal shares of the
//      (b, c, h) items.  The chunk's B tile (S x N) is loaded once and shared
//      by the heads that follow (B is the same for the heads of a group).
//      Per head the x tile (S x P) is scaled in shared memory by
//      w_s = exp(Acum_e - Acum_s) dt_s and
//        dH[c] = B^T (w o x)      (M = N = 128, N_mma = P = 64, K = S)
//      runs on the tensor core; dH (bf16) leaves by TMA tensor store.
//  state_pass_tc   states[c] = exp(Asum[c]) states[c-1] + dH[c] from the
//      stored bf16 memories, sequential in c; also writes the bf16 state
//      entering each chunk, hin[c] = bf16(states[c-1]) (hin[0] = init_state
//      or 0), the operand of the inter-chunk output product.
//  chunk_output    y = Y_diag + exp(Acum_t) Y_off with
//        G = C B^T,  P[t,s] = G[t,s] exp(Acum_t - Acum_s) dt_s (s <= t),
//        Y_diag = P x,  Y_off = C hin[c].
//      Persistent, one CTA per SM over cost-balanced ranges of the
//      (b, c, 128-row half, h) items.  G is computed once per (b, c, half,
//      group) into TMEM and shared by its heads; the P builders read it from TMEM
//      and write P (bf16) in 64-column panels, each handed to the MMA by its
//      own barrier pair.
//
// Decay factors: exp(Acum_t - Acum_s) = exp(Acum_t - Acum_r) exp(Acum_r -
// Acum_s) with r the first token of the 32-token column block holding s.  The
// column factor is at most exp(32 |a|max) dt_s, inside float range; the row
// factor is at most 1 and underflows only where the term is below about 2^-75
// of the diagonal's, which then counts as 0.  So one exponential per (row,
// block) and one per column are needed.
#include <cuda_bf16.h>
#include <string.h>

#include "dart_common.cuh"
#include "sm100.cuh"
#include "tensor_map.h"

namespace dart {
namespace {

using namespace sm100;

constexpr int kN = 128, kP = 64;
constexpr uint32_t kRowBytes = 128;                  // one 64-element bf16 row of a swizzle panel
constexpr uint32_t kBox = 128 * kRowBytes;           // a 128-row TMA box, 16 KB
constexpr int kScanMaxCtas = 160;                    // largest persistent grid (one CTA per SM)

struct ScanTcParams {
    CUtensorMap tmap_x;    // x  as (P, B*L, H), box (64, 128, 1)
    CUtensorMap tmap_b;    // Bm as (N, G, L, B), box (64, 1, 128, 1)
    CUtensorMap tmap_c;    // Cm as (N, G, L, B), box (64, 1, 128, 1)
    CUtensorMap tmap_hin;  // hin as (P, B*H*C*N), box (64, 128)
    CUtensorMap tmap_dh;   // dH as (P, B*H*C*N) bf16, box (64, 128): chunk_state's store
    CUtensorMap tmap_y;    // y as (P, H, L, B) fp32, box (32, 1, 128, 1): chunk_output's store
    const float* dt;
    const float* A;
    const float* init_state;
    __nv_bfloat16* dH;
    float* states;
    float* asum;
    __nv_bfloat16* hin;
    float* y;
    // per-token decay terms, each [B, H, C, S] fp32 (written by chunk_decay):
    //   a2   = log2(e) * Acum_s, the inclusive prefix of dt A inside the chunk
    //   colf = exp(Acum_r - Acum_s) dt_s, r the first token of s's 32-token block
    //   wst  = exp(Acum_end - Acum_s) dt_s, the weight of token s in dH[c]
    float* a2;
    float* colf;
    float* wst;
    int B, L, H, S, C;
    int G, HG;             // groups of heads sharing B and C, heads per group
    int co_range[kScanMaxCtas + 1];  // chunk_output: CTA r runs items co_range[r] .. co_range[r + 1] - 1
    int* status;
};

// ===========================================================================
// chunk_decay: the per-token decay terms of every (b, h, c).  One CTA per
// (b, c, group of 8 heads): the group's dt block [S tokens][8 heads] is read
// once (8 consecutive floats per token) into shared memory, head-major with
// one padding word per row; warp w then scans head w of the group in rounds
// of 32 tokens, one token per lane.
// ===========================================================================
template <int S>
__global__ void __launch_bounds__(256) chunk_decay_kernel(const __grid_constant__ ScanTcParams p) {
    constexpr int K = S / 32;             // rounds of 32 tokens
    __shared__ float dts[8 * (S + 1)];    // [head of the group][S + 1]
    griddep_wait();
    const int ngh = (p.H + 7) / 8;
    const int hgi = blockIdx.x % ngh;
    const int c = (blockIdx.x / ngh) % p.C, b = blockIdx.x / (ngh * p.C);
    const int nh = min(8, p.H - 8 * hgi);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = c * S;
    for (int i = threadIdx.x; i < 8 * S; i += blockDim.x) {
        const int t = i >> 3, hh = i & 7;
        // past the end of a partial last chunk (or of the heads): no decay, no input
        dts[hh * (S + 1) + t] =
            (t0 + t < p.L && hh < nh) ? p.dt[((size_t)b * p.L + t0 + t) * p.H + 8 * hgi + hh] : 0.f;
    }
    __syncthreads();
    if (warp >= nh) return;
    const int h = 8 * hgi + warp;
    const float Ah = p.A[h];
    const float* d = dts + warp * (S + 1);
    const size_t o = (((size_t)b * p.H + h) * p.C + c) * S;   // this (b, h, c) in the decay arrays
    float carry = 0.f;      // prefix of dt A over the previous rounds
    float v[K];
#pragma unroll
    for (int r = 0; r < K; ++r) {
        const float dv = d[32 * r + lane];
        float incl = dv * Ah;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float up = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += up;
        }
        v[r] = carry + incl;                                  // Acum at token 32 r + lane
        const float a2 = v[r] * kLog2e;
        const float a2r = __shfl_sync(0xffffffffu, a2, 0);    // the round's first token
        p.a2[o + 32 * r + lane] = a2;
        p.colf[o + 32 * r + lane] = exp2f(a2r - a2) * dv;
        carry = __shfl_sync(0xffffffffu, v[r], 31);
    }
    const float aend = carry;
#pragma unroll
    for (int r = 0; r < K; ++r) p.wst[o + 32 * r + lane] = expf(aend - v[r]) * d[32 * r + lane];
    if (lane == 0) p.asum[((size_t)b * p.H + h) * p.C + c] = aend;
}

// ===========================================================================
// chunk_state_tc
// ===========================================================================
namespace cs {
// warp 0 TMA, warp 1 MMA, warps 2-5 scale the x tiles, warps 6-9 write dH
constexpr int kThreads = 320;
constexpr int kScalers = 128, kEpi = 128;
constexpr int kMaxStages = 6;
enum Bar { B_FULL = 0, B_FREE = 1, X_FULL0 = 2, X_EMPTY0 = X_FULL0 + kMaxStages, W_READY0 = X_EMPTY0 + kMaxStages,
           ACC_FULL0 = W_READY0 + kMaxStages, ACC_EMPTY0 = ACC_FULL0 + 2, NUM_BARS = ACC_EMPTY0 + 2 };
static_assert(NUM_BARS == 24, "chunk_state barrier slots");

// Work items (b, c, h) in that order, h fastest; consecutive items of one
// (b, c) share the chunk's B tile.  CTA r of G takes items
// [r T / G, (r + 1) T / G): equal shares, and the B tile is reloaded only
// where the range crosses into the next chunk.
struct Item {
    int b, c, h;
};
__device__ __forceinline__ Item cs_item(const ScanTcParams& p, int j) {
    Item it;
    it.h = j % p.H;
    it.c = (j / p.H) % p.C;
    it.b = j / (p.H * p.C);
    return it;
}

// x tiles (S rows x 128 B) move through a ring of kStages buffers: loaded by
// TMA, scaled in place (row s times wst_s) by the scaler warps, consumed by
// the MMA.  The finished dH (bf16, 128 rows x 128 B) leaves through one of
// two swizzled staging tiles by TMA tensor store.
template <int S>
struct Layout {
    static constexpr int kStages = S == 256 ? 3 : 6;
    static_assert(kStages <= kMaxStages, "x ring depth");
    static constexpr uint32_t kOffB = 0;                        // 2 panels x S rows
    static constexpr uint32_t kOffX = 2 * S * kRowBytes;        // kStages buffers x S rows
    static constexpr uint32_t kXBytes = S * kRowBytes;
    static constexpr uint32_t kOffF = kOffX + kStages * kXBytes; // kStages buffers x wst[S] floats
    static constexpr uint32_t kOffOut = (kOffF + kStages * S * 4 + 1023) & ~1023u;   // 2 dH staging tiles
    static constexpr uint32_t kOffBar = kOffOut + 2 * kBox;
    static constexpr uint32_t kBytes = kOffBar + NUM_BARS * 8 + 16 + 1024;
    static_assert(kBytes <= 232448, "chunk_state shared memory");
};

template <int S>
__global__ void __launch_bounds__(kThreads, 1) chunk_state_tc_kernel(const __grid_constant__ ScanTcParams p) {
    using Ly = Layout<S>;
    constexpr int kSt = Ly::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const float* wst_s = reinterpret_cast<const float*>(smem + Ly::kOffF);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Ly::kOffBar + NUM_BARS * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    auto bar = [&](int i) -> uint32_t { return sbase + Ly::kOffBar + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int total = p.B * p.C * p.H;
    const int j0 = (int)((long long)blockIdx.x * total / gridDim.x);
    const int j1 = (int)((long long)(blockIdx.x + 1) * total / gridDim.x);
    const int n_items = j1 - j0;

    if (threadIdx.x == 0) {
        mbar_init(bar(B_FULL), 1);
        mbar_init(bar(B_FREE), 1);
        for (int s = 0; s < kSt; ++s) {
            mbar_init(bar(X_FULL0 + s), 1);
            mbar_init(bar(X_EMPTY0 + s), 1);
            mbar_init(bar(W_READY0 + s), kScalers / 32);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(bar(ACC_FULL0 + a), 1);
            mbar_init(bar(ACC_EMPTY0 + a), kEpi / 32);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    griddep_wait();

    const WaitCtx wc{abort_flag, p.status, 2};
    if (warp == 0) {
        // TMA: the whole warp walks the items, lane 0 issues
        if (lane == 0) {
            tma_prefetch_desc(&p.tmap_x);
            tma_prefetch_desc(&p.tmap_b);
        }
        int b_loads = 0;
        for (int i = 0; i < n_items; ++i) {
            const Item it = cs_item(p, j0 + i);
            const int t0 = it.c * S;                  // first token of the chunk
            if (i == 0 || it.h % p.HG == 0) {
                // a new chunk or group: its B tile, once the MMAs on the previous one are done
                if (b_loads > 0 && !mbar_wait_warp(bar(B_FREE), (uint32_t)(b_loads - 1) & 1u, wc, 7)) break;
                if (lane == 0) {
                    mbar_expect_tx(bar(B_FULL), 2 * S * kRowBytes);
                    for (int pnl = 0; pnl < 2; ++pnl)
                        for (int r = 0; r < S / 128; ++r)
                            tma_load_4d(sbase + Ly::kOffB + (uint32_t)pnl * S * kRowBytes + (uint32_t)r * kBox,
                                        &p.tmap_b, bar(B_FULL), 64 * pnl, it.h / p.HG, t0 + 128 * r, it.b);
                }
                ++b_loads;
            }
            const int xs = i % kSt;
            const uint32_t ph = (uint32_t)(i / kSt) & 1u;
            if (!mbar_wait_warp(bar(X_EMPTY0 + xs), ph ^ 1u, wc, 1)) break;
            if (lane == 0) {
                mbar_expect_tx(bar(X_FULL0 + xs), Ly::kXBytes + S * 4);
                for (int r = 0; r < S / 128; ++r)
                    tma_load_4d(sbase + Ly::kOffX + (uint32_t)xs * Ly::kXBytes + (uint32_t)r * kBox, &p.tmap_x,
                                bar(X_FULL0 + xs), 0, it.h, t0 + 128 * r, it.b);
                bulk_load(sbase + Ly::kOffF + (uint32_t)xs * S * 4,
                          p.wst + (((size_t)it.b * p.H + it.h) * p.C + it.c) * S, S * 4, bar(X_FULL0 + xs));
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // MMA: D[n, p] = sum_s B[s, n] W[s, p]: A = B^T (MN-major, M = n over
        // two 64-wide panels), B = W (MN-major), K = s.  Lane 0 issues.
        const uint32_t idesc = idesc_bf16_f32(128, kP, true, true);
        bool ok = true;
        int b_loads = 0;
        for (int i = 0; i < n_items && ok; ++i) {
            const Item it = cs_item(p, j0 + i);
            if (i == 0 || it.h % p.HG == 0) {
                if (!(ok = mbar_wait_warp(bar(B_FULL), (uint32_t)b_loads & 1u, wc, 2))) break;
                ++b_loads;
            }
            // the last item on this B tile releases it after its MMAs
            const bool last_on_b = i + 1 == n_items || (it.h + 1) % p.HG == 0;
            const int xs = i % kSt, a = i & 1;
            const uint32_t ph = (uint32_t)(i / kSt) & 1u;
            const uint32_t aph = (uint32_t)(i >> 1) & 1u;
            if (!(ok = mbar_wait_warp(bar(W_READY0 + xs), ph, wc, 3))) break;
            if (!(ok = mbar_wait_warp(bar(ACC_EMPTY0 + a), aph ^ 1u, wc, 4))) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t xbase = sbase + Ly::kOffX + (uint32_t)xs * Ly::kXBytes;
#pragma unroll 4
                for (int kk = 0; kk < S / 16; ++kk) {
                    const uint64_t ad = smem_desc_sw128(sbase + Ly::kOffB + (uint32_t)kk * 2048, S * kRowBytes, 1024);
                    const uint64_t bd = smem_desc_sw128(xbase + (uint32_t)kk * 2048, 8192, 1024);
                    mma_f16_ss(tmem + (uint32_t)a * 64, ad, bd, idesc, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(ACC_FULL0 + a));
                mma_commit(bar(X_EMPTY0 + xs));
                if (last_on_b) mma_commit(bar(B_FREE));
            }
            __syncwarp();
        }
    } else if (warp < 2 + kScalers / 32) {
        // ---------------------------------------------------------- scalers
        // row s of the x tile times wst_s, in place (bf16 -> fp32 -> bf16)
        const int wi = threadIdx.x - 64;            // 0..127
        bool ok = true;
        for (int i = 0; i < n_items && ok; ++i) {
            const int xs = i % kSt;
            const uint32_t ph = (uint32_t)(i / kSt) & 1u;
            if (!(ok = mbar_wait_warp(bar(X_FULL0 + xs), ph, wc, 6))) break;
            uint8_t* xb = smem + Ly::kOffX + (uint32_t)xs * Ly::kXBytes;
            const float* w = wst_s + xs * S;
#pragma unroll 4
            for (int k = wi; k < S * 8; k += kScalers) {
                uint4* ptr = reinterpret_cast<uint4*>(xb + (size_t)k * 16);
                float f[8];
                Vec16<__nv_bfloat16>::unpack(*ptr, f);
                const float ws = w[k >> 3];
#pragma unroll
                for (int j = 0; j < 8; ++j) f[j] *= ws;
                Vec16<__nv_bfloat16>::store(reinterpret_cast<__nv_bfloat16*>(ptr), f);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(W_READY0 + xs));
        }
    } else {
        // --------------------------------------------------------- epilogue
        // The four warps run every item's two named barriers whether or not
        // their own waits succeeded (they then skip the work), so none of
        // them can be left at a barrier the others never reach.
        const int wi = threadIdx.x - 64 - kScalers;  // 0..127
        const int quad = warp & 3;
        const int nrow = quad * 32 + lane;          // TMEM lane = state row n
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        bool ok = true;
        for (int i = 0; i < n_items; ++i) {
            const int a = i & 1;
            const uint32_t aph = (uint32_t)(i >> 1) & 1u;
            if (ok) ok = mbar_wait_warp(bar(ACC_FULL0 + a), aph, wc, 5);
            float v[kP];
            if (ok) {
                tc_fence_after();
                tmem_ld_32x32b_x32(t_lane + (uint32_t)a * 64, v);
                tmem_ld_32x32b_x32(t_lane + (uint32_t)a * 64 + 32, v + 32);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(ACC_EMPTY0 + a));
            }
            // staging tile i & 1 was last used by item i - 2: its store must
            // have finished reading it
            uint8_t* out_s = smem + Ly::kOffOut + (uint32_t)(i & 1) * kBox;
            if (wi == 0) bulk_wait_read<1>();
            named_bar_sync(1, kEpi);
            if (ok) {
                // row nrow, 16-byte chunk j at position j ^ (nrow & 7) of its 128-byte row
                uint8_t* drow = out_s + (uint32_t)nrow * kRowBytes;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    Vec16<__nv_bfloat16>::store(reinterpret_cast<__nv_bfloat16*>(drow + ((j ^ (nrow & 7)) << 4)), v + 8 * j);
            }
            fence_proxy_async_smem();
            named_bar_sync(1, kEpi);
            if (wi == 0 && !*abort_flag) {
                const Item it = cs_item(p, j0 + i);
                const int row = (((it.b * p.H + it.h) * p.C + it.c) * kN);
                tma_store_2d(&p.tmap_dh, smem_u32(out_s), 0, row);
                bulk_commit();
            }
        }
        if (wi == 0) bulk_wait<0>();  // stores complete before the CTA's shared memory goes away
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}
}  // namespace cs

// ===========================================================================
// state_pass_tc (CUDA cores; memory-bound)
// ===========================================================================
// states[c] = exp(Asum[c]) states[c-1] + dH[c] from the bf16 chunk memories
// chunk_state wrote, sequential in c, and hin[c] = bf16(states[c-1]).  Each
// thread owns 4 consecutive elements of one (b, h) state; the memories of the
// next kPre chunks are in flight while the current one is folded in, so the
// loads never wait on the dependent chain of FMAs.
constexpr int kPassPre = 8;
__global__ void __launch_bounds__(256) state_pass_tc_kernel(const __grid_constant__ ScanTcParams p) {
    constexpr int NP = kN * kP;
    griddep_wait();
    const int h = blockIdx.y, b = blockIdx.z;
    const int e4 = (blockIdx.x * blockDim.x + threadIdx.x) * 4;  // 4 consecutive elements
    if (e4 >= NP) return;
    const size_t bh = (size_t)b * p.H + h;
    const int C = p.C;
    float4 prev = p.init_state ? *reinterpret_cast<const float4*>(p.init_state + bh * NP + e4)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
    float* st = p.states + bh * (size_t)C * NP + e4;
    __nv_bfloat16* hin = p.hin + bh * (size_t)C * NP + e4;
    const uint2* dh = reinterpret_cast<const uint2*>(p.dH + bh * (size_t)C * NP + e4);
    const float* asum = p.asum + bh * C;
    uint2 pre[kPassPre];
#pragma unroll
    for (int q = 0; q < kPassPre; ++q) pre[q] = q < C ? __ldg(dh + (size_t)q * (NP / 4)) : make_uint2(0u, 0u);
    for (int c0 = 0; c0 < C; c0 += kPassPre) {
#pragma unroll
        for (int q = 0; q < kPassPre; ++q) {
            const int c = c0 + q;
            if (c < C) {
                const uint2 d = pre[q];
                if (c + kPassPre < C) pre[q] = __ldg(dh + (size_t)(c + kPassPre) * (NP / 4));
                __nv_bfloat162 lo = __floats2bfloat162_rn(prev.x, prev.y), hi = __floats2bfloat162_rn(prev.z, prev.w);
                uint2 pk;
                pk.x = *reinterpret_cast<uint32_t*>(&lo);
                pk.y = *reinterpret_cast<uint32_t*>(&hi);
                *reinterpret_cast<uint2*>(hin + (size_t)c * NP) = pk;
                const float dec = expf(__ldg(asum + c));
                prev = make_float4(fmaf(dec, prev.x, __uint_as_float(d.x << 16)),
                                   fmaf(dec, prev.y, __uint_as_float(d.x & 0xffff0000u)),
                                   fmaf(dec, prev.z, __uint_as_float(d.y << 16)),
                                   fmaf(dec, prev.w, __uint_as_float(d.y & 0xffff0000u)));
                *reinterpret_cast<float4*>(st + (size_t)c * NP) = prev;
            }
        }
    }
}

// ===========================================================================
// chunk_output_tc
// ===========================================================================
namespace co {
constexpr int kWorkers = 256;                  // warps 2-9 build P
constexpr int kEpi = 128;                      // warps 10-13 write y
constexpr int kThreads = 64 + kWorkers + kEpi; // warp 0 TMA, warp 1 MMA
// Barrier slots.  The two-deep rings take two consecutive slots; P is built
// and consumed in 64-column panels (at most four), each with its own
// ready / free pair, so the tensor core starts on a panel while the workers
// build the next one.  A group (b, c, half) shares C rows, B rows and G:
// GRP_FREE releases C, B and P after the group's last MMAs, G_FREE releases
// G after the P builders' last reads of it.
constexpr int kPanels = 4;
enum Bar { IN_FULL = 0, G_FULL = 1, G_FREE = 2, GRP_FREE = 3, X_FULL0 = 4, X_FREE0 = 6, P_READY0 = 8,
           P_FREE0 = P_READY0 + kPanels, ACC_FULL0 = P_FREE0 + kPanels, ACC_EMPTY0 = ACC_FULL0 + 2,
           NUM_BARS = ACC_EMPTY0 + 2 };
static_assert(NUM_BARS == 20, "barrier slots overlap");
constexpr uint32_t kOffC = 0;                          // C rows: 2 panels x 128 rows (32 KB)
constexpr uint32_t kOffBP = 2 * kBox;                  // B rows (2 panels x KS rows), later P (KS/64 panels x 128 rows)
constexpr uint32_t kOffX = kOffBP + 4 * kBox;          // 2 buffers x (256 rows x 128 B)
constexpr uint32_t kXBytes = 2 * kBox;
constexpr uint32_t kOffHp = kOffX + 2 * kXBytes;       // 2 buffers x 128 rows (16 KB)
constexpr uint32_t kOffF = kOffHp + 2 * kBox;          // 2 buffers x (a2[256], colf[256])
constexpr uint32_t kOffRs = kOffF + 2 * 2 * 256 * 4;  // row scales exp(Acum_t), ring of 4 items x 256
constexpr uint32_t kOffYs = kOffRs + 4 * 256 * 4;      // y staging: one box of 128 rows x 32 fp32 (16 KB)
constexpr uint32_t kOffBar = kOffYs + kBox;
constexpr uint32_t kBytes = kOffBar + NUM_BARS * 8 + 16 + 1024;
static_assert(kOffYs % 1024 == 0 && kBytes <= 232448, "chunk_output shared memory");
constexpr uint32_t kColDiag = 256, kColOff = 384;

// Work items (b, c, half, h), h fastest.  The items of one (b, c, half)
// form a group.  CTA r runs items co_range[r] .. co_range[r + 1] - 1.
struct Item {
    int b, c, half, h;
};
__device__ __forceinline__ Item co_item(const ScanTcParams& p, int j) {
    const int R = p.S / 128;
    const int g = j / p.H;
    Item it;
    it.h = j % p.H;
    it.half = g % R;
    it.c = (g / R) % p.C;
    it.b = g / (R * p.C);
    return it;
}

__global__ void __launch_bounds__(kThreads, 1) chunk_output_tc_kernel(const __grid_constant__ ScanTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const float* dec_s = reinterpret_cast<const float*>(smem + kOffF);  // [2][a2[256], colf[256]]
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffBar + NUM_BARS * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.S;
    const int j0 = p.co_range[blockIdx.x];
    const int n_items = p.co_range[blockIdx.x + 1] - j0;
    // a group shares C rows, B rows and G: one (b, c, half) and one group of heads
    auto group_first = [&](int i, const Item& it) { return i == 0 || it.h % p.HG == 0; };
    auto group_last = [&](int i, const Item& it) { return i + 1 == n_items || (it.h + 1) % p.HG == 0; };

    if (threadIdx.x == 0) {
        mbar_init(bar(IN_FULL), 1);
        mbar_init(bar(G_FULL), 1);
        mbar_init(bar(G_FREE), kWorkers / 32);
        mbar_init(bar(GRP_FREE), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(X_FULL0 + s), 1);
            mbar_init(bar(X_FREE0 + s), 1);
            mbar_init(bar(ACC_FULL0 + s), 1);
            mbar_init(bar(ACC_EMPTY0 + s), kEpi / 32);
        }
        for (int k = 0; k < kPanels; ++k) {
            mbar_init(bar(P_READY0 + k), kWorkers / 32);
            mbar_init(bar(P_FREE0 + k), 1);
        }
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
    griddep_wait();

    const WaitCtx wc{abort_flag, p.status, 3};
    if (warp == 0) {
        // TMA: the whole warp walks the items, lane 0 issues
        if (lane == 0) {
            tma_prefetch_desc(&p.tmap_x);
            tma_prefetch_desc(&p.tmap_b);
            tma_prefetch_desc(&p.tmap_c);
            tma_prefetch_desc(&p.tmap_hin);
        }
        int ng = 0;  // groups loaded so far
        for (int i = 0; i < n_items; ++i) {
            const Item it = co_item(p, j0 + i);
            const int KS = 128 * (it.half + 1);            // source tokens this half depends on
            const int t0 = it.c * S;                       // first token of the chunk
            const bool has_off = (it.c > 0) || (p.init_state != nullptr);
            if (group_first(i, it)) {
                // C rows of this half (A of G and of Y_off) and B rows 0..KS-1 (B of G),
                // once the previous group's MMAs are done with C, B and P
                if (ng > 0 && !mbar_wait_warp(bar(GRP_FREE), (uint32_t)(ng - 1) & 1u, wc, 10)) break;
                if (lane == 0) {
                    mbar_expect_tx(bar(IN_FULL), 2 * kBox + 2 * (uint32_t)KS * kRowBytes);
                    for (int pnl = 0; pnl < 2; ++pnl) {
                        tma_load_4d(sbase + kOffC + (uint32_t)pnl * kBox, &p.tmap_c, bar(IN_FULL), 64 * pnl,
                                    it.h / p.HG, t0 + 128 * it.half, it.b);
                        for (int r = 0; r < KS / 128; ++r)
                            tma_load_4d(sbase + kOffBP + (uint32_t)pnl * KS * kRowBytes + (uint32_t)r * kBox,
                                        &p.tmap_b, bar(IN_FULL), 64 * pnl, it.h / p.HG, t0 + 128 * r, it.b);
                    }
                }
                ++ng;
            }
            const int xs = i & 1;
            const uint32_t ph = (uint32_t)(i >> 1) & 1u;
            if (!mbar_wait_warp(bar(X_FREE0 + xs), ph ^ 1u, wc, 1)) break;
            if (lane == 0) {
                const uint32_t bytes = (uint32_t)KS * kRowBytes + (has_off ? kBox : 0u) + 2u * KS * 4u;
                mbar_expect_tx(bar(X_FULL0 + xs), bytes);
                const size_t drow = (((size_t)it.b * p.H + it.h) * p.C + it.c) * S;   // (b, h, c) in the decay arrays
                bulk_load(sbase + kOffF + (uint32_t)xs * 2048, p.a2 + drow, KS * 4, bar(X_FULL0 + xs));
                bulk_load(sbase + kOffF + (uint32_t)xs * 2048 + 1024, p.colf + drow, KS * 4, bar(X_FULL0 + xs));
                for (int r = 0; r < KS / 128; ++r)
                    tma_load_4d(sbase + kOffX + (uint32_t)xs * kXBytes + (uint32_t)r * kBox, &p.tmap_x,
                                bar(X_FULL0 + xs), 0, it.h, t0 + 128 * r, it.b);
                if (has_off)
                    tma_load_2d(sbase + kOffHp + (uint32_t)xs * kBox, &p.tmap_hin, bar(X_FULL0 + xs), 0,
                                ((it.b * p.H + it.h) * p.C + it.c) * kN);
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // MMA: lane 0 issues, the whole warp walks the items
        const uint32_t idesc_y = idesc_bf16_f32(128, kP, false, true);
        bool ok = true;
        int ng = 0;
        uint32_t ready_par = 0;  // bit k: parity of the next P_READY(k) completion
        for (int i = 0; i < n_items && ok; ++i) {
            const Item it = co_item(p, j0 + i);
            const int KS = 128 * (it.half + 1);
            const int npanel = KS / 64;
            const bool has_off = (it.c > 0) || (p.init_state != nullptr);
            if (group_first(i, it)) {
                // G[t, s] = sum_n C[t, n] B[s, n]: both K-major, K = N; written over the
                // previous group's G once the P builders are done reading it
                if (!(ok = mbar_wait_warp(bar(IN_FULL), (uint32_t)ng & 1u, wc, 2))) break;
                if (ng > 0 && !(ok = mbar_wait_warp(bar(G_FREE), (uint32_t)(ng - 1) & 1u, wc, 11))) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t idesc_g = idesc_bf16_f32(128, KS, false, false);
#pragma unroll
                    for (int kk = 0; kk < kN / 16; ++kk) {
                        const uint32_t koff = (uint32_t)(kk & 3) * 32;   // 16 K-elements inside a panel
                        const uint64_t ad = smem_desc_sw128(sbase + kOffC + (uint32_t)(kk >> 2) * kBox + koff, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(
                            sbase + kOffBP + (uint32_t)(kk >> 2) * (uint32_t)KS * kRowBytes + koff, 16, 1024);
                        mma_f16_ss(tmem, ad, bd, idesc_g, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(G_FULL));
                }
                __syncwarp();
                ++ng;
            }
            const int xs = i & 1, a = i & 1;
            const uint32_t ph = (uint32_t)(i >> 1) & 1u;
            if (!(ok = mbar_wait_warp(bar(X_FULL0 + xs), ph, wc, 5))) break;
            if (!(ok = mbar_wait_warp(bar(ACC_EMPTY0 + a), ph ^ 1u, wc, 4))) break;
            tc_fence_after();
            if (has_off && lane == 0) {
                // Y_off = C hin[c]: A = C rows (K-major, K = n), B = hin (MN-major); needs no P
                const uint32_t hbase = sbase + kOffHp + (uint32_t)xs * kBox;
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk) {
                    const uint64_t ad = smem_desc_sw128(
                        sbase + kOffC + (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(hbase + (uint32_t)kk * 2048, 8192, 1024);
                    mma_f16_ss(tmem + kColOff + (uint32_t)a * 64, ad, bd, idesc_y, kk > 0 ? 1u : 0u);
                }
            }
            __syncwarp();
            // Y_diag = P x with dt folded into P: A = P (K-major, K = s), B = x (MN-major),
            // one 64-column panel of P at a time
            const uint32_t xbase = sbase + kOffX + (uint32_t)xs * kXBytes;
            for (int k = 0; k < npanel && ok; ++k) {
                if (!(ok = mbar_wait_warp(bar(P_READY0 + k), (ready_par >> k) & 1u, wc, 3))) break;
                ready_par ^= 1u << k;
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int kk = 4 * k + k4;
                        const uint64_t ad = smem_desc_sw128(sbase + kOffBP + (uint32_t)k * kBox + (uint32_t)k4 * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(xbase + (uint32_t)kk * 2048, 8192, 1024);
                        mma_f16_ss(tmem + kColDiag + (uint32_t)a * 64, ad, bd, idesc_y, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(P_FREE0 + k));
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) {
                mma_commit(bar(ACC_FULL0 + a));
                mma_commit(bar(X_FREE0 + xs));
                if (group_last(i, it)) mma_commit(bar(GRP_FREE));
            }
            __syncwarp();
        }
    } else if (warp >= 2 + kWorkers / 32) {
        // --------------------------------------------------------- epilogue
        // y = Y_diag + exp(Acum_t) Y_off for the item whose accumulators are
        // ready, one box of 32 columns at a time: written 128-byte-swizzled
        // into the staging area and stored by TMA.  The four warps run every
        // box's named barriers, also after a failed wait (they then skip the
        // work).
        const int quad = warp & 3;
        const int trow = quad * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        const bool issuer = warp == 2 + kWorkers / 32 && lane == 0;
        uint8_t* yrow = smem + kOffYs + (uint32_t)trow * kRowBytes;
        const float* rs_s = reinterpret_cast<const float*>(smem + kOffRs);
        bool ok = true;
        for (int i = 0; i < n_items; ++i) {
            const Item it = co_item(p, j0 + i);
            const bool has_off = (it.c > 0) || (p.init_state != nullptr);
            const int a = i & 1;
            const uint32_t ph = (uint32_t)(i >> 1) & 1u;
            if (ok) ok = mbar_wait_warp(bar(ACC_FULL0 + a), ph, wc, 8);
            float yv[64];
            if (ok) {
                tc_fence_after();
                // exp(Acum_t), left by the P builders: the decay terms in the x
                // buffer may already belong to a later item
                const float row_scale = rs_s[(i & 3) * 256 + 128 * it.half + trow];
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    float yo[32];
                    tmem_ld_32x32b_x32(t_lane + kColDiag + (uint32_t)a * 64 + (uint32_t)ch * 32, yv + 32 * ch);
                    if (has_off) tmem_ld_32x32b_x32(t_lane + kColOff + (uint32_t)a * 64 + (uint32_t)ch * 32, yo);
                    tmem_ld_wait();
                    if (has_off) {
#pragma unroll
                        for (int q = 0; q < 32; ++q) yv[32 * ch + q] = fmaf(row_scale, yo[q], yv[32 * ch + q]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(ACC_EMPTY0 + a));
            }
            const int t0 = it.c * S;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                if (issuer) bulk_wait_read<0>();   // the previous box has left the staging area
                named_bar_sync(1, kEpi);
                if (ok) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4*>(yrow + ((q ^ (trow & 7)) << 4)) =
                            make_float4(yv[32 * ch + 4 * q], yv[32 * ch + 4 * q + 1], yv[32 * ch + 4 * q + 2],
                                        yv[32 * ch + 4 * q + 3]);
                }
                fence_proxy_async_smem();
                named_bar_sync(1, kEpi);
                if (issuer && !*abort_flag && t0 + 128 * it.half < p.L) {   // rows past the end are not written
                    tma_store_4d(&p.tmap_y, sbase + kOffYs, 32 * ch, it.h, t0 + 128 * it.half, it.b);
                    bulk_commit();
                }
            }
        }
        if (issuer) bulk_wait<0>();   // y written before the CTA's shared memory goes away
    } else {
        // ---------------------------------------------------------- P build
        const int wk = warp - 2;                         // 0..7
        const int quad = warp & 3;                       // TMEM lane quadrant
        const int colhalf = wk >> 2;                     // which half of the columns
        const int trow = quad * 32 + lane;               // row inside the half (TMEM lane)
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        float* rs_w = reinterpret_cast<float*>(smem + kOffRs);
        bool ok = true;
        int ng = 0;
        uint32_t free_cnt = 0;  // bit k: parity of the P_FREE(k) commits made for earlier items
        for (int i = 0; i < n_items; ++i) {
            const Item it = co_item(p, j0 + i);
            const int KS = 128 * (it.half + 1);
            const int npanel = KS / 64;                  // 64-column panels of P; this warp builds
                                                         // block 2k + colhalf of panel k
            const int t = 128 * it.half + trow;          // chunk-local token of this row
            const bool first = group_first(i, it);
            // decay terms of this item arrive with its x tile
            const int xs = i & 1;
            const uint32_t ph = (uint32_t)(i >> 1) & 1u;
            if (ok) ok = mbar_wait_warp(bar(X_FULL0 + xs), ph, wc, 9);
            const float* a2 = dec_s + xs * 512;
            const float* colf = a2 + 256;
            const float a2t = ok ? a2[t] : 0.f;
            // The epilogue reads item i's row scale after item i's MMAs; the
            // slot is rewritten by item i + 4, whose P build cannot start
            // before the epilogue has released item i's accumulators.
            if (colhalf == 0) rs_w[(i & 3) * 256 + t] = exp2f(a2t);
            // a new group's P may be written once its G is in TMEM (the P
            // buffer held its B rows until then)
            if (first) {
                if (ok) ok = mbar_wait_warp(bar(G_FULL), (uint32_t)ng & 1u, wc, 6);
                ++ng;
            }
            const int warp_tmin = 128 * it.half + 32 * quad;     // first row of this warp
            const int warp_tmax = warp_tmin + 31;                // last row of this warp
            for (int k = 0; k < npanel; ++k) {
                // within a group, panel k may be written once the previous
                // item's MMA on it is done
                if (ok && !first) ok = mbar_wait_warp(bar(P_FREE0 + k), ((free_cnt >> k) & 1u) ^ 1u, wc, 7);
                if (!ok) break;
                tc_fence_after();
                const int j = 2 * k + colhalf;
                const int s0 = 32 * j;
                uint32_t packed[16];
                if (s0 <= warp_tmax) {                           // warp-uniform
                    float g[32];
                    tmem_ld_32x32b_x32(t_lane + (uint32_t)s0, g);
                    float2 cf[16];                               // column factors, same for every row
                    const float4* c4 = reinterpret_cast<const float4*>(colf + s0);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 v = c4[q];
                        cf[2 * q] = make_float2(v.x, v.y);
                        cf[2 * q + 1] = make_float2(v.z, v.w);
                    }
                    const float rf = exp2f(a2t - a2[s0]);
                    const float2 rf2 = make_float2(rf, rf);
                    tmem_ld_wait();
                    if (s0 + 31 <= warp_tmin) {                  // block below every row's diagonal
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            const float2 v = __fmul2_rn(__fmul2_rn(make_float2(g[2 * q], g[2 * q + 1]), cf[q]), rf2);
                            __nv_bfloat162 pr = __floats2bfloat162_rn(v.x, v.y);
                            packed[q] = *reinterpret_cast<uint32_t*>(&pr);
                        }
                    } else {                                     // the diagonal block: causal mask s <= t
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            const int sa = s0 + 2 * q;
                            const float2 v = __fmul2_rn(__fmul2_rn(make_float2(g[2 * q], g[2 * q + 1]), cf[q]), rf2);
                            __nv_bfloat162 pr = __floats2bfloat162_rn(sa <= t ? v.x : 0.f, sa + 1 <= t ? v.y : 0.f);
                            packed[q] = *reinterpret_cast<uint32_t*>(&pr);
                        }
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) packed[q] = 0u;
                }
                // row trow of panel k, 16-byte chunks colhalf*4 .. +3, 128-byte swizzle
                uint8_t* prow = smem + kOffBP + (uint32_t)k * kBox + (uint32_t)trow * kRowBytes;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int ch = (colhalf * 4 + u) ^ (trow & 7);
                    *reinterpret_cast<uint4*>(prow + ch * 16) =
                        make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
                }
                tc_fence_before();
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(P_READY0 + k));
            }
            free_cnt ^= (1u << npanel) - 1u;   // the MMA commits P_FREE(k) once for this item, k < npanel
            // after the group's last item the P builders are done with its G
            if (group_last(i, it) && lane == 0) mbar_arrive(bar(G_FREE));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}
}  // namespace co

// Token-indexed tensors are described with the sequence and batch axes
// apart, so a box that runs past the end of a partial last chunk reads
// zeros and writes nothing there (instead of reaching the next sequence).
bool make_maps(const ScanArgs& a, ScanTcParams& p) {
    const int C = (a.L + a.S - 1) / a.S;
    {
        const uint64_t dims[4] = {(uint64_t)kP, (uint64_t)a.H, (uint64_t)a.L, (uint64_t)a.B};
        const uint64_t strides[3] = {(uint64_t)kP * 2, (uint64_t)a.H * kP * 2, (uint64_t)a.L * a.H * kP * 2};
        const uint32_t box[4] = {64, 1, 128, 1};
        if (!encode_tile_map_bf16(&p.tmap_x, 4, a.x, dims, strides, box)) return false;
    }
    {
        const uint64_t dims[4] = {(uint64_t)kN, (uint64_t)a.G, (uint64_t)a.L, (uint64_t)a.B};
        const uint64_t strides[3] = {(uint64_t)kN * 2, (uint64_t)a.G * kN * 2, (uint64_t)a.L * a.G * kN * 2};
        const uint32_t box[4] = {64, 1, 128, 1};
        if (!encode_tile_map_bf16(&p.tmap_b, 4, a.Bm, dims, strides, box)) return false;
        if (!encode_tile_map_bf16(&p.tmap_c, 4, a.Cm, dims, strides, box)) return false;
    }
    {
        const uint64_t dims[2] = {(uint64_t)kP, (uint64_t)a.B * a.H * C * kN};
        const uint64_t strides[1] = {(uint64_t)kP * 2};
        const uint32_t box[2] = {64, 128};
        if (!encode_tile_map_bf16(&p.tmap_hin, 2, a.hin, dims, strides, box)) return false;
        if (!encode_tile_map_bf16(&p.tmap_dh, 2, a.dH, dims, strides, box)) return false;
    }
    {
        const uint64_t dims[4] = {(uint64_t)kP, (uint64_t)a.H, (uint64_t)a.L, (uint64_t)a.B};
        const uint64_t strides[3] = {(uint64_t)kP * 4, (uint64_t)a.H * kP * 4, (uint64_t)a.L * a.H * kP * 4};
        const uint32_t box[4] = {32, 1, 128, 1};
        if (!encode_tile_map_f32(&p.tmap_y, 4, a.y, dims, strides, box)) return false;
    }
    return true;
}

}  // namespace

bool ssd_scan_tc_applicable(int N, int P, int S, dart_dtype dt) {
    return dt == DART_BF16 && N == kN && P == kP && (S == 128 || S == 256);
}

cudaError_t launch_ssd_scan_tc(const ScanArgs& a, cudaStream_t st) {
    ScanTcParams p;
    memset(&p, 0, sizeof(p));
    if (!make_maps(a, p)) return cudaErrorInvalidValue;
    p.dt = a.dt;
    p.A = a.A;
    p.init_state = a.init_state;
    p.dH = static_cast<__nv_bfloat16*>(a.dH);
    p.states = a.states;
    p.asum = a.asum;
    p.hin = static_cast<__nv_bfloat16*>(a.hin);
    p.y = a.y;
    p.B = a.B; p.L = a.L; p.H = a.H; p.S = a.S; p.C = (a.L + a.S - 1) / a.S;
    p.G = a.G; p.HG = a.H / a.G;
    const size_t bhcs = (size_t)a.B * a.H * p.C * a.S;   // decay arrays are [B, H, C, S]
    p.a2 = a.decay;
    p.colf = a.decay + bhcs;
    p.wst = a.decay + 2 * bhcs;
    p.status = a.status;
    cudaError_t e;
    // 0. per-token decay terms, one CTA per (b, c, group of 8 heads)
    {
        const int grid = a.B * p.C * ((a.H + 7) / 8);
        e = a.S == 256 ? launch_dependent(chunk_decay_kernel<256>, dim3(grid), dim3(256), 0, st, 1, p)
                       : launch_dependent(chunk_decay_kernel<128>, dim3(grid), dim3(256), 0, st, 1, p);
        if (e != cudaSuccess) return e;
    }
    // 1. chunk memories
    {
        // persistent: one CTA per SM, equal shares of the (b, c, h) items
        const int sms = sm_count();
        if (sms <= 0) return cudaErrorInvalidDevice;
        const int items = a.B * p.C * a.H;
        const int grid = items < sms ? items : sms;
        if (a.S == 256) {
            auto k = cs::chunk_state_tc_kernel<256>;
            const uint32_t smem = cs::Layout<256>::kBytes;
            if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
                return e;
            if ((e = launch_dependent(k, dim3(grid), dim3(cs::kThreads), smem, st, 1, p)) != cudaSuccess) return e;
        } else {
            auto k = cs::chunk_state_tc_kernel<128>;
            const uint32_t smem = cs::Layout<128>::kBytes;
            if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
                return e;
            if ((e = launch_dependent(k, dim3(grid), dim3(cs::kThreads), smem, st, 1, p)) != cudaSuccess) return e;
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // 2. state passing
    if ((e = launch_dependent(state_pass_tc_kernel, dim3(kN * kP / 4 / 256, a.H, a.B), dim3(256), 0, st, 1, p)) !=
        cudaSuccess)
        return e;
    // 3. outputs
    {
        // persistent: one CTA per SM, contiguous ranges of the (b, c, half, h)
        // items with equal estimated work.  Building P bounds an item, and on
        // the busiest TMEM lane quadrant an item of the second half (256
        // source tokens) has twice the blocks of one of the first; a group
        // change (C and B rows, G) costs about one first-half item.
        const int sms = sm_count();
        if (sms <= 0) return cudaErrorInvalidDevice;
        const int R = a.S / 128;
        const int items = a.B * p.C * R * a.H;
        int grid = sms < kScanMaxCtas ? sms : kScanMaxCtas;
        if (items < grid) grid = items;
        auto cost = [&](int j) {
            const int half = (j / a.H) % R;
            return (half == 0 ? 2 : 4) + ((j % a.H) % (a.H / a.G) == 0 ? 2 : 0);
        };
        long long total = 0;
        for (int j = 0; j < items; ++j) total += cost(j);
        long long acc = 0;
        int r = 1;
        p.co_range[0] = 0;
        for (int j = 0; j < items && r < grid; ++j) {
            acc += cost(j);
            while (r < grid && acc * grid >= total * r) p.co_range[r++] = j + 1;
        }
        while (r <= grid) p.co_range[r++] = items;
        if ((e = cudaFuncSetAttribute(co::chunk_output_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)co::kBytes)) != cudaSuccess)
            return e;
        if ((e = launch_dependent(co::chunk_output_tc_kernel, dim3(grid), dim3(co::kThreads), co::kBytes, st, 1, p)) !=
            cudaSuccess)
            return e;
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    count_launches(4);
    return cudaSuccess;
}

}  // namespace dart
