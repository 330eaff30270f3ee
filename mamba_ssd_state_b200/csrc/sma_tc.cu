// sma_tc.cu -- state-memory attention on the 5th-generation tensor cores.
//
// What it computes (Pith review of DART, "Core claim" / "What carries the
// argument"; SMA Eqs. (5)-(10)): for token t in chunk k(t) and each earlier
// chunk memory c < k(t),
//   U_{t,c} = Q_t^T dH[c]  (P),   V_{t,c} = C_t^T dH[c]  (P),
//   s_{t,c} = U_{t,c} . E_t / sqrt(N)   (= Q_t . (dH[c] E_t) / sqrt(N)),
//   o_t = sum_c softmax_c(s) V_{t,c},   out = y_ssd + g o_t.
//
// Why this shape: the only dense contractions are [Q_T; C_T] x dH[c]; the
// "PV" step is per token and per chunk (every token decodes its own value),
// so it is element-wise work on CUDA cores, not a second GEMM.  One CTA owns
// a tile of 128 query tokens of one (b, h), all inside chunk k:
//   A operands  Q_T, C_T   128 x 128 bf16, K-major, loaded once per tile;
//   B operand   4 chunk memories side by side, 128 (K = N) x 256 (4 x P),
//               MN-major exactly as stored in HBM, streamed by TMA;
//   D           U (TMEM columns 0..255) and V (columns 256..511), fp32.
// Each batch of 4 memories costs two M=128, N=256, K=128 MMAs.  The epilogue
// warps read U as soon as it lands (scores, online softmax) and hand the U
// columns back while the V MMA runs, then read V (value accumulation) while
// the next batch's U MMA runs.
//
// Roles (320 threads): warp 0 issues TMA, warp 1 allocates TMEM and issues
// tcgen05.mma, warps 2-9 run the epilogue as four pairs, one pair per TMEM
// lane quadrant (32 token rows); the two warps of a pair split the 64 value
// columns, exchange partial scores through shared memory, run the same
// online softmax and each write their half of the output row.  Splitting
// the columns halves the epilogue's time per batch, which is what keeps the
// MMA fed.  The grid is persistent: CTA i takes tiles i, i+G, ... of a list
// ordered from the most memories to the fewest, so the triangular work
// spreads evenly.
//
// CTA pairs (S a multiple of 256): two CTAs of a cluster run the two
// 128-token halves of a 256-token tile as one M = 256 MMA (tcgen05 with
// cta_group::2).  Each CTA loads its own Q and C rows and two of the four
// memories of a batch (its half of N), so the 128 KB memory ring holds four
// stages instead of two and each SM streams half the memory bytes; CTA 0
// issues the MMAs and owns the FULL / EMPTY barriers they wait on, the
// peer's loads complete on them and its epilogue warps arrive on them
// remotely; the commits reach both CTAs.  S = 128 runs one CTA per tile.
//
// Decayed memories (kDecay; referee comment 3 on Eq. (8)): memory c reaches
// token t scaled by w = exp(sum_{r=e(c)+1}^{t} dt_r A_h), and since U and V are
// linear in the memory the scale is applied in the epilogue: score w s, value
// weight p w (the softmax normaliser keeps p).  The base-2 exponent comes from
// the per-token and per-chunk prefixes of sma_decay.cu.
#include <cuda_bf16.h>
#include <string.h>

#include <atomic>

#include "dart_common.cuh"
#include "sm100.cuh"
#include "tensor_map.h"

namespace dart {
namespace {

using namespace sm100;

constexpr int kN = 128, kP = 64;   // compiled shape
constexpr int kBQ = 128;           // query tokens per tile (MMA M)
constexpr int kCB = 4;             // chunk memories per MMA (N = 4 * P = 256)
constexpr uint32_t kHalfA = 128 * 64 * 2;        // 128 rows x 64 bf16 (one swizzle panel)
constexpr uint32_t kMemBytes = kN * kP * 2;       // one chunk memory, 16 KB
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffC = 2 * kHalfA;
constexpr uint32_t kOffB = 4 * kHalfA;
constexpr uint32_t kRingBytes = 2 * kCB * kMemBytes;   // the memory ring: 128 KB
// Ring geometry.  A single CTA holds all four memories of a batch (two
// stages of 64 KB); in a CTA pair each CTA holds two of them (its half of
// the MMA's N columns), so the same 128 KB give four stages.
template <bool kPair>
struct Ring {
    static constexpr int kMem = kPair ? 2 : 4;
    static constexpr int kStages = kPair ? 4 : 2;
    static constexpr uint32_t kStageBytes = kMem * kMemBytes;
    static_assert(kStages * kStageBytes == kRingBytes, "ring size");
};
constexpr int kMaxStages = 4;
// Output tile: at a tile end the gated attention output g o / l of the 128
// rows, as two 128-byte-swizzled boxes of 32 fp32 columns (the layout of the
// out tensor map), added into out (which holds y_ssd) by a TMA reduction.
// While a tile runs, its first 8 KB hold the partial-score exchange
// [2 parity][2 half][128 rows][4].
constexpr uint32_t kOffO = kOffB + kRingBytes;
constexpr uint32_t kOBox = 128 * 32 * 4;              // one box: 128 rows x 32 fp32
constexpr uint32_t kOffBar = kOffO + 2 * kOBox;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // + alignment slack
constexpr int kEpiWarps = 8;                          // four pairs, one pair per TMEM lane quadrant
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColV = 256;
constexpr int kHalfP = kP / 2;                        // value columns per epilogue warp

// Barrier slots (explicit; the memory ring takes consecutive slots).
enum Bar { Q_FULL = 0, Q_FREE = 1, C_FULL = 2, C_FREE = 3, U_FULL = 4, U_EMPTY = 5, V_FULL = 6, V_EMPTY = 7,
           B_FULL0 = 8, B_EMPTY0 = B_FULL0 + kMaxStages, NUM_BARS = B_EMPTY0 + kMaxStages };
static_assert(NUM_BARS * 8 + 8 <= 256, "barrier block");
static_assert(kOffO % 1024 == 0 && 2 * 2 * 128 * 4 * 4 <= 2 * kOBox && kSmemBytes <= 232448,
              "shared memory layout");

struct SmaTcParams {
    // Token-indexed tensors keep the sequence and batch axes apart, so a tile
    // that runs past the end of a partial last chunk reads zeros and writes
    // nothing there.
    CUtensorMap tmap_q;  // Q viewed as dims (N, H, L, B), box (64, 1, 128, 1)
    CUtensorMap tmap_c;  // Cm viewed as dims (N, G, L, B), box (64, 1, 128, 1)
    CUtensorMap tmap_h;  // dH viewed as dims (P, B*H*C*N)
    CUtensorMap tmap_e;  // E viewed as dims (P, H, L, B), box (64, 1, 128, 1): L2 prefetch only
    CUtensorMap tmap_o;  // out viewed as dims (P, H, L, B) fp32, box (32, 1, 128, 1): reduce-add / store
    const __nv_bfloat16* E;
    const float* y_ssd;
    float* out;
    const float* la2;     // decayed memories: [B,H,C*S] in-chunk log2-decay prefix
    const double* gpre;   // decayed memories: [B,H,C] chunk-level prefix
    float g;
    int add_into_out;  // 1: out already holds y_ssd, the tile end adds g o / l; 0: it stores o / l
    int B, L, H, S, C;
    int HG;            // heads per group sharing C (head h reads group h / HG)
    int cta_per_tile;  // 1, or 2 for a CTA pair (each CTA 128 of the tile's 256 rows)
    int tiles_per_chunk, total_tiles;
    int* status;
};

struct Tile {
    int b, h, k, t0;
};

// Tile list ordered by decreasing chunk index (most memories first).
// `rank` picks this CTA's 128 rows of a pair tile.
__device__ __forceinline__ Tile decode_tile(const SmaTcParams& p, int i, int rank) {
    const int per_k = p.B * p.H * p.tiles_per_chunk;
    Tile t;
    t.k = p.C - 1 - i / per_k;
    const int r = i % per_k;
    const int sub = r % p.tiles_per_chunk;
    const int bh = r / p.tiles_per_chunk;
    t.b = bh / p.H;
    t.h = bh % p.H;
    t.t0 = t.k * p.S + (sub * p.cta_per_tile + rank) * kBQ;
    return t;
}

template <bool kPair, bool kDecay>
__global__ void __launch_bounds__(kThreads, 1) sma_tc_kernel(const __grid_constant__ SmaTcParams p) {
    using Rg = Ring<kPair>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffBar + NUM_BARS * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // A pair tile is run by both CTAs of a cluster; CTA 0 issues the MMAs
    // and owns the FULL / EMPTY barriers they wait on.
    const int rank = kPair ? (int)cluster_ctarank() : 0;
    const int tile0 = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int tstride = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    auto bar_lead = [&](int i) -> uint32_t { return kPair ? mapa_shared(bar(i), 0) : bar(i); };

    if (threadIdx.x == 0) {
        mbar_init(bar(Q_FULL), 1);
        mbar_init(bar(Q_FREE), 1);
        mbar_init(bar(C_FULL), 1);
        mbar_init(bar(C_FREE), 1);
        mbar_init(bar(U_FULL), 1);
        mbar_init(bar(U_EMPTY), kEpiWarps * (kPair ? 2 : 1));
        mbar_init(bar(V_FULL), 1);
        mbar_init(bar(V_EMPTY), kEpiWarps * (kPair ? 2 : 1));
        for (int s = 0; s < Rg::kStages; ++s) {
            mbar_init(bar(B_FULL0 + s), 1);
            mbar_init(bar(B_EMPTY0 + s), 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tmap_q);
        tma_prefetch_desc(&p.tmap_c);
        tma_prefetch_desc(&p.tmap_h);
        tma_prefetch_desc(&p.tmap_e);
        tma_prefetch_desc(&p.tmap_o);
    }
    if (warp == 1) {
        if (kPair) {
            tmem_alloc_pair(smem_u32(tmem_holder), kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_holder), kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if (kPair)
        cluster_sync();  // both CTAs' barriers exist before any remote arrive or copy
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    griddep_wait();

    const WaitCtx wc{abort_flag, p.status, 1};
    if (warp == 0) {
        // ------------------------------------------------------------ TMA
        // The whole warp walks the schedule; lane 0 issues the copies.
        uint32_t q_ph = 0, c_ph = 0;
        int it_b = 0;
        bool ok = true;
        auto load_b = [&](const Tile& t, int j) -> bool {
            const int nv = min(kCB, t.k - kCB * j);
            const int s = it_b % Rg::kStages;
            const uint32_t ph = (uint32_t)(it_b / Rg::kStages) & 1u;
            if (!mbar_wait_warp(bar(B_EMPTY0 + s), ph ^ 1, wc, 3)) return false;
            if (lane == 0) {
                // this CTA's memories of the batch: all four, or its two of a pair
                const int q0 = Rg::kMem * rank;
                const int mine = max(0, min(Rg::kMem, nv - q0));
                if (rank == 0) mbar_expect_tx(bar(B_FULL0 + s), (uint32_t)nv * kMemBytes);
                const int mem_row = ((t.b * p.H + t.h) * p.C + kCB * j + q0) * kN;
                const uint32_t dst = sbase + kOffB + (uint32_t)s * Rg::kStageBytes;
                for (int q = 0; q < mine; ++q) {
                    if (kPair)
                        tma_load_2d_pair(dst + (uint32_t)q * kMemBytes, &p.tmap_h, bar_lead(B_FULL0 + s), 0,
                                         mem_row + q * kN);
                    else
                        tma_load_2d(dst + (uint32_t)q * kMemBytes, &p.tmap_h, bar(B_FULL0 + s), 0, mem_row + q * kN);
                }
            }
            ++it_b;
            return true;
        };
        for (int i = tile0; i < p.total_tiles && ok; i += tstride) {
            const Tile t = decode_tile(p, i, rank);
            if (t.k == 0) continue;
            const int row = t.t0;   // first token of the tile within sequence t.b
            // The first memories of this tile go out before its Q and C: their
            // stage is free long before the previous tile releases Q and C.
            if (!(ok = load_b(t, 0))) break;
            if (!(ok = mbar_wait_warp(bar(Q_FREE), q_ph ^ 1, wc, 1))) break;
            if (lane == 0) {
                if (rank == 0) mbar_expect_tx(bar(Q_FULL), 2 * kHalfA * (kPair ? 2 : 1));
                if (kPair) {
                    tma_load_4d_pair(sbase + kOffQ, &p.tmap_q, bar_lead(Q_FULL), 0, t.h, row, t.b);
                    tma_load_4d_pair(sbase + kOffQ + kHalfA, &p.tmap_q, bar_lead(Q_FULL), 64, t.h, row, t.b);
                } else {
                    tma_load_4d(sbase + kOffQ, &p.tmap_q, bar(Q_FULL), 0, t.h, row, t.b);
                    tma_load_4d(sbase + kOffQ + kHalfA, &p.tmap_q, bar(Q_FULL), 64, t.h, row, t.b);
                }
            }
            q_ph ^= 1;
            if (!(ok = mbar_wait_warp(bar(C_FREE), c_ph ^ 1, wc, 2))) break;
            if (lane == 0) {
                if (rank == 0) mbar_expect_tx(bar(C_FULL), 2 * kHalfA * (kPair ? 2 : 1));
                if (kPair) {
                    tma_load_4d_pair(sbase + kOffC, &p.tmap_c, bar_lead(C_FULL), 0, t.h / p.HG, row, t.b);
                    tma_load_4d_pair(sbase + kOffC + kHalfA, &p.tmap_c, bar_lead(C_FULL), 64, t.h / p.HG, row, t.b);
                } else {
                    tma_load_4d(sbase + kOffC, &p.tmap_c, bar(C_FULL), 0, t.h / p.HG, row, t.b);
                    tma_load_4d(sbase + kOffC + kHalfA, &p.tmap_c, bar(C_FULL), 64, t.h / p.HG, row, t.b);
                }
                // the next tile's rows start moving into L2 now: its Q and C
                // (if it has memories), the E rows its epilogue starts from
                // and the out rows (holding y_ssd) its output is added into
                if (i + tstride < p.total_tiles) {
                    const Tile tn = decode_tile(p, i + tstride, rank);
                    const int rown = tn.t0;
                    if (tn.k > 0) {
                        tma_prefetch_4d(&p.tmap_q, 0, tn.h, rown, tn.b);
                        tma_prefetch_4d(&p.tmap_q, 64, tn.h, rown, tn.b);
                        tma_prefetch_4d(&p.tmap_c, 0, tn.h / p.HG, rown, tn.b);
                        tma_prefetch_4d(&p.tmap_c, 64, tn.h / p.HG, rown, tn.b);
                        tma_prefetch_4d(&p.tmap_e, 0, tn.h, rown, tn.b);
                    }
                    if (p.add_into_out && tn.k > 0) {
                        tma_prefetch_4d(&p.tmap_o, 0, tn.h, rown, tn.b);
                        tma_prefetch_4d(&p.tmap_o, 32, tn.h, rown, tn.b);
                    }
                }
            }
            c_ph ^= 1;
            const int nbatch = (t.k + kCB - 1) / kCB;
            for (int j = 1; j < nbatch; ++j)
                if (!(ok = load_b(t, j))) break;
            __syncwarp();
        }
    } else if (warp == 1 && rank == 0) {
        // ------------------------------------------------------------ MMA
        // The whole warp walks the schedule; lane 0 issues the MMAs (in a
        // pair, the leader's for both CTAs: M = 256, N = 256 with each CTA
        // supplying its two memories, commits reaching both CTAs).
        uint32_t q_ph = 0, c_ph = 0;
        int it_b = 0, it_u = 0;
        bool ok = true;
        auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc) {
            if (kPair)
                mma_f16_ss_pair(d, ad, bd, idesc, acc);
            else
                mma_f16_ss(d, ad, bd, idesc, acc);
        };
        auto commit = [&](int b) {
            if (kPair)
                mma_commit_pair(bar(b));
            else
                mma_commit(bar(b));
        };
        for (int i = tile0; i < p.total_tiles && ok; i += tstride) {
            const Tile t = decode_tile(p, i, rank);
            if (t.k == 0) continue;
            if (!(ok = mbar_wait_warp(bar(Q_FULL), q_ph, wc, 4))) break;
            q_ph ^= 1;
            tc_fence_after();
            const int nbatch = (t.k + kCB - 1) / kCB;
            for (int j = 0; j < nbatch; ++j, ++it_b, ++it_u) {
                const int nv = min(kCB, t.k - kCB * j);
                const int s = it_b % Rg::kStages;
                const uint32_t ph = (uint32_t)(it_b / Rg::kStages) & 1u;
                // a pair always multiplies all four column blocks (the epilogue
                // reads only the nv valid ones); N splits evenly over the CTAs
                const uint32_t idesc = kPair ? idesc_bf16_f32(2 * kBQ, kP * kCB, false, true)
                                             : idesc_bf16_f32(kBQ, kP * nv, false, true);
                const uint32_t b_base = sbase + kOffB + (uint32_t)s * Rg::kStageBytes;
                if (!(ok = mbar_wait_warp(bar(B_FULL0 + s), ph, wc, 5))) break;
                if (!(ok = mbar_wait_warp(bar(U_EMPTY), ((uint32_t)it_u & 1u) ^ 1u, wc, 6))) break;
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < kN / 16; ++kk) {
                        const uint64_t ad = smem_desc_sw128(sbase + kOffQ + (uint32_t)(kk >> 2) * kHalfA + (uint32_t)(kk & 3) * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(b_base + (uint32_t)kk * 2048, kMemBytes, 1024);
                        mma(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
                    }
                    commit(U_FULL);
                    if (j == nbatch - 1) commit(Q_FREE);
                }
                __syncwarp();
                if (j == 0) {
                    if (!(ok = mbar_wait_warp(bar(C_FULL), c_ph, wc, 7))) break;
                    c_ph ^= 1;
                }
                if (!(ok = mbar_wait_warp(bar(V_EMPTY), ((uint32_t)it_u & 1u) ^ 1u, wc, 8))) break;
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < kN / 16; ++kk) {
                        const uint64_t ad = smem_desc_sw128(sbase + kOffC + (uint32_t)(kk >> 2) * kHalfA + (uint32_t)(kk & 3) * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(b_base + (uint32_t)kk * 2048, kMemBytes, 1024);
                        mma(tmem + kColV, ad, bd, idesc, kk > 0 ? 1u : 0u);
                    }
                    commit(V_FULL);
                    commit(B_EMPTY0 + s);
                    if (j == nbatch - 1) commit(C_FREE);
                }
                __syncwarp();
            }
        }
    } else if (warp >= 2) {
        // ------------------------------------------------------- epilogue
        // Warp pair (w, w+4) shares TMEM lane quadrant w & 3 (32 token rows);
        // warp half h owns value columns [32h, 32h+32) of every memory.  Both
        // warps of a pair run the same batches and the same named barrier
        // per batch, also after a failed wait (they then skip the work).
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const int col0 = half * kHalfP;
        const int row = quad * 32 + lane;          // token row inside the tile
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        const float sscale = kLog2e * rsqrtf((float)kN);
        float* xbuf = reinterpret_cast<float*>(smem + kOffO);
        // this lane's row of the output tile: box `half`, row `row`, 128-byte swizzle
        uint8_t* orow_s = smem + kOffO + (uint32_t)half * kOBox + (uint32_t)row * 128u;
        const bool issuer = warp == 2 && lane == 0;  // issues the output tile's TMA operation
        // The eight epilogue warps meet at named barrier 1 before the output
        // tile is written, after it is written, and before the first score
        // exchange of every tile (after the issuer saw the previous tile's
        // TMA operation finish reading the tile).  All of them run every
        // tile and batch, also after a failed wait.
        auto tile_sync = [&]() { named_bar_sync(1, 32 * kEpiWarps); };
        int it_u = 0;
        bool ok = true;
        auto row_offset = [&](const Tile& t) -> size_t {
            const size_t tok = (size_t)t.b * p.L + t.t0 + row;
            return (tok * p.H + t.h) * kP + col0;
        };
        // This warp's 32 columns of E for the tile about to run, as packed
        // bf16; the next tile's are fetched at the end of each tile.
        uint4 e_raw[kHalfP / 8];
        auto load_e = [&](int i) {
#pragma unroll
            for (int q = 0; q < kHalfP / 8; ++q) e_raw[q] = make_uint4(0u, 0u, 0u, 0u);
            if (i >= p.total_tiles) return;
            const Tile t = decode_tile(p, i, rank);
            if (t.k == 0 || t.t0 + row >= p.L) return;   // no memories, or a row past the end of the sequence
            const uint4* src = reinterpret_cast<const uint4*>(p.E + row_offset(t));
#pragma unroll
            for (int q = 0; q < kHalfP / 8; ++q) e_raw[q] = __ldg(src + q);
        };
        load_e(tile0);
        for (int i = tile0; i < p.total_tiles; i += tstride) {
            const Tile t = decode_tile(p, i, rank);
            float2 o2[kHalfP / 2];
#pragma unroll
            for (int j = 0; j < kHalfP / 2; ++j) o2[j] = make_float2(0.f, 0.f);
            float l = 0.f;
            if (t.k > 0) {
                // E widened to fp32 once per tile (bf16 -> fp32 is a shift)
                float2 e2[kHalfP / 2];
                {
#pragma unroll
                    for (int q = 0; q < kHalfP / 8; ++q) {
                        const uint4 v4 = e_raw[q];
                        const uint32_t w4[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                        for (int r = 0; r < 4; ++r)
                            e2[4 * q + r] = make_float2(__uint_as_float(w4[r] << 16), __uint_as_float(w4[r] & 0xffff0000u));
                    }
                }
                float m = -INFINITY;
                const int nbatch = (t.k + kCB - 1) / kCB;
                // decayed memories: this row's in-chunk prefix and the chunk prefix at k
                const size_t bh = (size_t)t.b * p.H + t.h;
                float la_row = 0.f;
                double g_k = 0.0;
                if (kDecay) {
                    la_row = p.la2[bh * p.C * p.S + t.t0 + row];   // t0 + row < C * S
                    g_k = p.gpre[bh * p.C + t.k];
                }
                for (int j = 0; j < nbatch; ++j, ++it_u) {
                    const int nv = min(kCB, t.k - kCB * j);
                    const uint32_t ph = (uint32_t)it_u & 1u;
                    float part[kCB] = {0.f, 0.f, 0.f, 0.f};
                    float wd[kCB] = {1.f, 1.f, 1.f, 1.f};   // decay of each memory at this row
                    if (kDecay) {
#pragma unroll
                        for (int c = 0; c < kCB; ++c)
                            if (c < nv)   // memory kCB j + c < k, so its index + 1 <= k < C
                                wd[c] = exp2f(la_row + (float)(g_k - __ldg(p.gpre + bh * p.C + kCB * j + c + 1)));
                    }
                    if (ok) ok = mbar_wait_warp(bar(U_FULL), ph, wc, 9);
                    if (ok) {
                        tc_fence_after();
#pragma unroll
                        for (int c = 0; c < kCB; ++c) {
                            if (c < nv) {
                                float u[kHalfP];
                                tmem_ld_32x32b_x32(t_lane + (uint32_t)(c * kP + col0), u);
                                tmem_ld_wait();
                                float2 a0 = make_float2(0.f, 0.f), a1 = a0;
#pragma unroll
                                for (int q = 0; q < kHalfP / 2; q += 2) {
                                    a0 = __ffma2_rn(make_float2(u[2 * q], u[2 * q + 1]), e2[q], a0);
                                    a1 = __ffma2_rn(make_float2(u[2 * q + 2], u[2 * q + 3]), e2[q + 1], a1);
                                }
                                part[c] = (a0.x + a1.x) + (a0.y + a1.y);
                            }
                        }
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if (kPair)
                                mbar_arrive_cluster(bar_lead(U_EMPTY));
                            else
                                mbar_arrive(bar(U_EMPTY));
                        }
                    }
                    if (j == 0) {  // the exchange area is free once the last tile's output left it
                        if (issuer) bulk_wait_read<0>();
                        tile_sync();
                    }
                    // scores: own partial + partner's partial
                    float* xs = xbuf + (((it_u & 1) * 2 + half) * 128 + row) * 4;
                    const float* xp = xbuf + (((it_u & 1) * 2 + (1 - half)) * 128 + row) * 4;
                    *reinterpret_cast<float4*>(xs) = make_float4(part[0], part[1], part[2], part[3]);
                    named_bar_sync(2 + quad, 64);
                    const float4 pp = *reinterpret_cast<const float4*>(xp);
                    const float other[kCB] = {pp.x, pp.y, pp.z, pp.w};
                    float sc[kCB];
#pragma unroll
                    for (int c = 0; c < kCB; ++c) sc[c] = c < nv ? (part[c] + other[c]) * sscale * wd[c] : -INFINITY;
                    float mnew = m;
#pragma unroll
                    for (int c = 0; c < kCB; ++c) mnew = fmaxf(mnew, sc[c]);
                    const float alpha = exp2f(m - mnew);
                    float w[kCB];
#pragma unroll
                    for (int c = 0; c < kCB; ++c) w[c] = c < nv ? exp2f(sc[c] - mnew) : 0.f;
                    l = l * alpha + (w[0] + w[1]) + (w[2] + w[3]);
                    m = mnew;
                    const float2 alpha2 = make_float2(alpha, alpha);
#pragma unroll
                    for (int q = 0; q < kHalfP / 2; ++q) o2[q] = __fmul2_rn(o2[q], alpha2);
                    if (ok) ok = mbar_wait_warp(bar(V_FULL), ph, wc, 10);
                    if (ok) {
                        tc_fence_after();
#pragma unroll
                        for (int c = 0; c < kCB; ++c) {
                            if (c < nv) {
                                float v[kHalfP];
                                tmem_ld_32x32b_x32(t_lane + kColV + (uint32_t)(c * kP + col0), v);
                                tmem_ld_wait();
                                const float wv = kDecay ? w[c] * wd[c] : w[c];
                                const float2 w2 = make_float2(wv, wv);
#pragma unroll
                                for (int q = 0; q < kHalfP / 2; ++q)
                                    o2[q] = __ffma2_rn(w2, make_float2(v[2 * q], v[2 * q + 1]), o2[q]);
                            }
                        }
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if (kPair)
                                mbar_arrive_cluster(bar_lead(V_EMPTY));
                            else
                                mbar_arrive(bar(V_EMPTY));
                        }
                    }
                }
            }
            const float inv = t.k > 0 && l > 0.f ? 1.f / l : 0.f;
            // Tile end.  The next tile's E row goes out first (its latency
            // overlaps the rest); then every lane writes g o / l of its row
            // and 32 columns into the output tile and one thread hands the
            // tile to the TMA unit, which adds it into out (holding y_ssd)
            // or stores it.  No lane touches y_ssd or out itself.
            const bool next_mem = i + tstride < p.total_tiles && decode_tile(p, i + tstride, rank).k > 0 &&
                                  decode_tile(p, i + tstride, rank).t0 + row < p.L;
            uint4 en[kHalfP / 8];
            if (next_mem) {
                const uint4* src = reinterpret_cast<const uint4*>(p.E + row_offset(decode_tile(p, i + tstride, rank)));
#pragma unroll
                for (int q = 0; q < kHalfP / 8; ++q) en[q] = __ldg(src + q);
            } else {
#pragma unroll
                for (int q = 0; q < kHalfP / 8; ++q) en[q] = make_uint4(0u, 0u, 0u, 0u);
            }
            if (issuer) bulk_wait_read<0>();   // a tile without memories has no exchange step
            tile_sync();                        // exchange area no longer read
            const float gi = (p.add_into_out ? p.g : 1.f) * inv;
#pragma unroll
            for (int q = 0; q < kHalfP / 4; ++q) {
                const float2 lo = o2[2 * q], hi = o2[2 * q + 1];
                *reinterpret_cast<float4*>(orow_s + (((uint32_t)q ^ (uint32_t)(row & 7)) << 4)) =
                    make_float4(gi * lo.x, gi * lo.y, gi * hi.x, gi * hi.y);
            }
            fence_proxy_async_smem();
            tile_sync();
            // (a tile without memories adds nothing: out already holds y_ssd there;
            // a tile that starts past the end of the sequence has no rows to write)
            if (issuer && !*abort_flag && (t.k > 0 || !p.add_into_out) && t.t0 < p.L) {
                if (p.add_into_out) {
                    tma_reduce_add_4d(&p.tmap_o, sbase + kOffO, 0, t.h, t.t0, t.b);
                    tma_reduce_add_4d(&p.tmap_o, sbase + kOffO + kOBox, 32, t.h, t.t0, t.b);
                } else {
                    tma_store_4d(&p.tmap_o, sbase + kOffO, 0, t.h, t.t0, t.b);
                    tma_store_4d(&p.tmap_o, sbase + kOffO + kOBox, 32, t.h, t.t0, t.b);
                }
                bulk_commit();
            }
#pragma unroll
            for (int q = 0; q < kHalfP / 8; ++q) e_raw[q] = en[q];
        }
        if (issuer) bulk_wait<0>();  // out written before the CTA's shared memory goes away
    }

    tc_fence_before();
    if (kPair)
        cluster_sync();  // neither CTA leaves while the other may still reach its memory
    else
        __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        if (kPair)
            tmem_dealloc_pair(tmem, kTmemCols);
        else
            tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool sma_tc_applicable(int N, int P, int S, dart_dtype dt) {
    return dt == DART_BF16 && N == kN && P == kP && S % kBQ == 0;
}

cudaError_t launch_sma_tc(const SmaArgs& a, cudaStream_t st) {
    SmaTcParams p;
    memset(&p, 0, sizeof(p));
    const int C = (a.L + a.S - 1) / a.S;   // a partial last chunk counts
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
    {
        const uint64_t dims[4] = {(uint64_t)kP, (uint64_t)a.H, (uint64_t)a.L, (uint64_t)a.B};
        const uint64_t strides[3] = {(uint64_t)kP * 2, (uint64_t)a.H * kP * 2, (uint64_t)a.L * a.H * kP * 2};
        const uint32_t box[4] = {64, 1, kBQ, 1};
        if (!encode_tile_map_bf16(&p.tmap_e, 4, a.E, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[4] = {(uint64_t)kP, (uint64_t)a.H, (uint64_t)a.L, (uint64_t)a.B};
        const uint64_t strides[3] = {(uint64_t)kP * 4, (uint64_t)a.H * kP * 4, (uint64_t)a.L * a.H * kP * 4};
        const uint32_t box[4] = {32, 1, kBQ, 1};
        if (!encode_tile_map_f32(&p.tmap_o, 4, a.out, dims, strides, box)) return cudaErrorInvalidValue;
    }
    p.E = static_cast<const __nv_bfloat16*>(a.E);
    p.la2 = a.la2;
    p.gpre = a.gpre;
    const bool decayed = a.la2 != nullptr;
    p.y_ssd = a.y_ssd;
    p.out = a.out;
    p.g = a.g;
    // The kernel adds g o into out, so out must hold y_ssd first; with no
    // y_ssd it stores o itself.
    p.add_into_out = a.y_ssd != nullptr;
    if (a.y_ssd && a.y_ssd != a.out) {
        const size_t bytes = (size_t)a.B * a.L * a.H * kP * sizeof(float);
        cudaError_t ce = cudaMemcpyAsync(a.out, a.y_ssd, bytes, cudaMemcpyDeviceToDevice, st);
        if (ce != cudaSuccess) return ce;
    }
    p.B = a.B; p.L = a.L; p.H = a.H; p.S = a.S; p.C = C;
    p.HG = a.H / a.G;
    p.status = a.status;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    cudaError_t e;
    if (a.S % (2 * kBQ) == 0) {
        // CTA pairs: each pair tile covers 256 query rows of one (b, h, chunk)
        p.cta_per_tile = 2;
        p.tiles_per_chunk = a.S / (2 * kBQ);
        p.total_tiles = C * a.B * a.H * p.tiles_per_chunk;
        auto kern = decayed ? sma_tc_kernel<true, true> : sma_tc_kernel<true, false>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes)) != cudaSuccess)
            return e;
        cudaLaunchConfig_t cfg;
        memset(&cfg, 0, sizeof(cfg));
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        // it may start while the previous launch on the stream finishes; the
        // kernel waits for it before touching global memory
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kSmemBytes;
        cfg.stream = st;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        // as many pairs as can be resident at once (not every SM need pair
        // up), queried once per device and variant; threads that race on the
        // first query store the same value
        static std::atomic<int> pairs_cache[2][64];
        int dev = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        int clusters = dev >= 0 && dev < 64 ? pairs_cache[decayed][dev].load(std::memory_order_relaxed) : 0;
        if (clusters <= 0) {
            cfg.gridDim = dim3(2 * (unsigned)(sms / 2), 1, 1);
            if ((e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg)) != cudaSuccess) return e;
            if (clusters <= 0) return cudaErrorInvalidConfiguration;
            if (dev >= 0 && dev < 64) pairs_cache[decayed][dev].store(clusters, std::memory_order_relaxed);
        }
        if (clusters > p.total_tiles) clusters = p.total_tiles;
        cfg.gridDim = dim3(2 * (unsigned)clusters, 1, 1);
        cfg.numAttrs = 2;
        if ((e = cudaLaunchKernelEx(&cfg, kern, p)) != cudaSuccess) return e;
    } else {
        p.cta_per_tile = 1;
        p.tiles_per_chunk = a.S / kBQ;
        p.total_tiles = C * a.B * a.H * p.tiles_per_chunk;
        const int grid = p.total_tiles < sms ? p.total_tiles : sms;
        auto kern = decayed ? sma_tc_kernel<false, true> : sma_tc_kernel<false, false>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes)) != cudaSuccess)
            return e;
        if ((e = launch_dependent(kern, dim3(grid), dim3(kThreads), kSmemBytes, st, 1, p)) != cudaSuccess) return e;
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launches(1);
    return cudaSuccess;
}

}  // namespace dart
