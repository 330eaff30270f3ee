// dart_abi.cu -- the extern "C" surface declared in include/dart.h:
// host-side validation, workspace sizing, dispatch to the kernel families and
// the device status word.
#include <atomic>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "dart_backward.cuh"

namespace dart {
// [0]: status flags; [1]: (kernel id << 8 | wait site) of the first bounded
// wait that gave up, 0 if none.
__device__ int g_status[2] = {0, 0};

namespace {
std::atomic<unsigned long long> g_launches{0};
}  // namespace

void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }
}  // namespace dart

namespace {

// Device address of the status word on the current device, looked up once
// per device.  Threads that race on the first lookup store the same value.
int* status_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    static std::atomic<int*> cache[64];
    int* w = cache[dev].load(std::memory_order_relaxed);
    if (!w) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, dart::g_status) != cudaSuccess) return nullptr;
        w = static_cast<int*>(p);
        cache[dev].store(w, std::memory_order_relaxed);
    }
    return w;
}

thread_local char t_err[512] = "";

dart_status fail(dart_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_err, sizeof(t_err), fmt, ap);
    va_end(ap);
    return st;
}

dart_status cuda_fail(cudaError_t e, const char* where) {
    return fail(DART_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace of the scan: per-chunk decay sums (float), padded to 256 bytes,
// followed on the tensor-core path by the bf16 state entering each chunk.
size_t scan_asum_bytes(size_t bhc) { return (bhc * sizeof(float) + 255) & ~size_t(255); }

#define DART_REQUIRE_PTR(p)                                                           \
    do {                                                                              \
        if (!(p)) return fail(DART_ERR_INVALID_ARG, "%s: null pointer", #p);          \
        if (!aligned16(p)) return fail(DART_ERR_INVALID_ARG, "%s: not 16-byte aligned", #p); \
    } while (0)

#define DART_OPTIONAL_PTR(p)                                                          \
    do {                                                                              \
        if ((p) && !aligned16(p))                                                     \
            return fail(DART_ERR_INVALID_ARG, "%s: not 16-byte aligned", #p);         \
    } while (0)

dart_status check_common(const dart_dims* d, dart_dtype dt, bool need_seqlen) {
    if (!d) return fail(DART_ERR_INVALID_ARG, "dims: null pointer");
    if (dt != DART_F32 && dt != DART_BF16) return fail(DART_ERR_INVALID_ARG, "dtype: unknown value %d", (int)dt);
    if (d->batch < 1 || d->nheads < 1 || d->headdim < 1 || d->dstate < 1 || d->chunk < 1)
        return fail(DART_ERR_INVALID_ARG, "dims: batch, nheads, headdim, dstate and chunk must be >= 1");
    if (d->ngroups < 1 || d->nheads % d->ngroups != 0)
        return fail(DART_ERR_INVALID_ARG, "ngroups = %d: must be >= 1 and divide nheads = %d", d->ngroups, d->nheads);
    if (need_seqlen) {
        if (d->seqlen < 1) return fail(DART_ERR_INVALID_ARG, "dims: seqlen must be >= 1");
    }
    if (d->batch > 65535 || d->nheads > 65535)
        return fail(DART_ERR_UNSUPPORTED, "batch and nheads must be <= 65535");
    return DART_OK;
}

}  // namespace

extern "C" {

int dart_abi_version(void) { return 4; }

unsigned long long dart_launch_count(void) { return dart::g_launches.load(std::memory_order_relaxed); }

const char* dart_last_error(void) { return t_err; }

int dart_supported(int dstate, int headdim, int chunk, dart_dtype dtype) {
    if (dtype != DART_F32 && dtype != DART_BF16) return 0;
    return dart::ssd_scan_supported(dstate, headdim, chunk, dtype) &&
           dart::sma_supported(dstate, headdim, chunk, dtype) &&
           dart::decode_supported(dstate, headdim, chunk, dtype);
}

const char* dart_sma_impl(int dstate, int headdim, int chunk, dart_dtype dtype) {
    if ((dtype != DART_F32 && dtype != DART_BF16) || !dart::sma_supported(dstate, headdim, chunk, dtype))
        return "";
    return dart::sma_impl_name(dstate, headdim, chunk, dtype);
}

size_t dart_ssd_chunk_scan_workspace_bytes(const dart_dims* d, dart_dtype dtype) {
    if (!d || d->chunk < 1) return 0;
    const size_t C = (size_t)((d->seqlen + d->chunk - 1) / d->chunk);
    const size_t bhc = (size_t)d->batch * (size_t)d->nheads * C;
    size_t bytes = scan_asum_bytes(bhc);
    if (dart::ssd_scan_tc_applicable(d->dstate, d->headdim, d->chunk, dtype)) {
        bytes += bhc * (size_t)d->dstate * (size_t)d->headdim * 2;  // bf16 state entering each chunk
        bytes += 3 * bhc * (size_t)d->chunk * sizeof(float);         // per-token decay terms
    }
    return bytes;
}

dart_status dart_ssd_chunk_scan(const dart_dims* d, dart_dtype dtype, const void* x, const float* dt,
                                const float* A, const void* Bm, const void* Cm, const float* init_state,
                                float* y_ssd, void* dH, float* states, void* workspace,
                                size_t workspace_bytes, void* stream) {
    t_err[0] = 0;
    dart_status st = check_common(d, dtype, true);
    if (st != DART_OK) return st;
    if (!dart::ssd_scan_supported(d->dstate, d->headdim, d->chunk, dtype))
        return fail(DART_ERR_UNSUPPORTED, "dart_ssd_chunk_scan: (N=%d, P=%d, S=%d) not compiled",
                    d->dstate, d->headdim, d->chunk);
    DART_REQUIRE_PTR(x); DART_REQUIRE_PTR(dt); DART_REQUIRE_PTR(A); DART_REQUIRE_PTR(Bm);
    DART_REQUIRE_PTR(Cm); DART_OPTIONAL_PTR(init_state); DART_REQUIRE_PTR(y_ssd);
    DART_REQUIRE_PTR(dH); DART_REQUIRE_PTR(states); DART_REQUIRE_PTR(workspace);
    if (workspace_bytes < dart_ssd_chunk_scan_workspace_bytes(d, dtype))
        return fail(DART_ERR_INVALID_ARG, "workspace: %zu bytes, need %zu", workspace_bytes,
                    dart_ssd_chunk_scan_workspace_bytes(d, dtype));
    const size_t bhc = (size_t)d->batch * (size_t)d->nheads * (size_t)((d->seqlen + d->chunk - 1) / d->chunk);
    char* hin = static_cast<char*>(workspace) + scan_asum_bytes(bhc);
    float* decay = reinterpret_cast<float*>(hin + bhc * (size_t)d->dstate * (size_t)d->headdim * 2);
    dart::ScanArgs a{d->batch, d->seqlen, d->nheads, d->headdim, d->dstate, d->chunk, d->ngroups,
                     x, dt, A, Bm, Cm, init_state, y_ssd, dH, states, static_cast<float*>(workspace),
                     hin, decay, status_word()};
    if (!a.status) return fail(DART_ERR_CUDA, "dart_ssd_chunk_scan: no device status word");
    cudaError_t e = dart::launch_ssd_scan(a, dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dart_ssd_chunk_scan launch");
    return DART_OK;
}

dart_status dart_sma_forward(const dart_dims* d, dart_dtype dtype, const void* Q, const void* E,
                             const void* Cm, const void* dH, float g, const float* y_ssd, float* out,
                             void* stream) {
    t_err[0] = 0;
    dart_status st = check_common(d, dtype, true);
    if (st != DART_OK) return st;
    if (!dart::sma_supported(d->dstate, d->headdim, d->chunk, dtype))
        return fail(DART_ERR_UNSUPPORTED, "dart_sma_forward: (N=%d, P=%d, S=%d) not compiled",
                    d->dstate, d->headdim, d->chunk);
    DART_REQUIRE_PTR(Q); DART_REQUIRE_PTR(E); DART_REQUIRE_PTR(Cm); DART_REQUIRE_PTR(dH);
    DART_OPTIONAL_PTR(y_ssd); DART_REQUIRE_PTR(out);
    if (y_ssd && y_ssd != out) {
        const size_t bytes = (size_t)d->batch * d->seqlen * d->nheads * d->headdim * sizeof(float);
        const uintptr_t ya = reinterpret_cast<uintptr_t>(y_ssd), oa = reinterpret_cast<uintptr_t>(out);
        if (ya < oa + bytes && oa < ya + bytes)
            return fail(DART_ERR_INVALID_ARG, "dart_sma_forward: out overlaps y_ssd without being the same pointer");
    }
    dart::SmaArgs a{d->batch, d->seqlen, d->nheads, d->headdim, d->dstate, d->chunk, d->ngroups,
                    Q, E, Cm, dH, g, y_ssd, out, status_word()};
    if (!a.status) return fail(DART_ERR_CUDA, "dart_sma_forward: no device status word");
    cudaError_t e = dart::launch_sma(a, dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dart_sma_forward launch");
    return DART_OK;
}

size_t dart_sma_decayed_workspace_bytes(const dart_dims* d) {
    if (!d) return 0;
    return dart::sma_decay_workspace_bytes(d->batch, d->seqlen, d->nheads, d->chunk);
}

dart_status dart_sma_forward_decayed(const dart_dims* d, dart_dtype dtype, const void* Q, const void* E,
                                     const void* Cm, const void* dH, const float* dt, const float* A, float g,
                                     const float* y_ssd, float* out, void* workspace, size_t workspace_bytes,
                                     void* stream) {
    t_err[0] = 0;
    dart_status st = check_common(d, dtype, true);
    if (st != DART_OK) return st;
    if (!dart::sma_supported(d->dstate, d->headdim, d->chunk, dtype))
        return fail(DART_ERR_UNSUPPORTED, "dart_sma_forward_decayed: (N=%d, P=%d, S=%d) not compiled",
                    d->dstate, d->headdim, d->chunk);
    DART_REQUIRE_PTR(Q); DART_REQUIRE_PTR(E); DART_REQUIRE_PTR(Cm); DART_REQUIRE_PTR(dH);
    DART_REQUIRE_PTR(dt); DART_REQUIRE_PTR(A);
    DART_OPTIONAL_PTR(y_ssd); DART_REQUIRE_PTR(out); DART_REQUIRE_PTR(workspace);
    if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0)
        return fail(DART_ERR_INVALID_ARG, "dart_sma_forward_decayed: workspace not 16-byte aligned");
    const size_t need = dart_sma_decayed_workspace_bytes(d);
    if (workspace_bytes < need)
        return fail(DART_ERR_INVALID_ARG, "workspace: %zu bytes, need %zu", workspace_bytes, need);
    if (y_ssd && y_ssd != out) {
        const size_t bytes = (size_t)d->batch * d->seqlen * d->nheads * d->headdim * sizeof(float);
        const uintptr_t ya = reinterpret_cast<uintptr_t>(y_ssd), oa = reinterpret_cast<uintptr_t>(out);
        if (ya < oa + bytes && oa < ya + bytes)
            return fail(DART_ERR_INVALID_ARG,
                        "dart_sma_forward_decayed: out overlaps y_ssd without being the same pointer");
    }
    const int C = (d->seqlen + d->chunk - 1) / d->chunk;
    float* la2 = static_cast<float*>(workspace);
    const size_t la2_bytes = ((sizeof(float) * (size_t)d->batch * d->nheads * C * d->chunk) + 255) & ~size_t(255);
    double* gpre = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + la2_bytes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = dart::launch_sma_decay_terms(d->batch, d->seqlen, d->nheads, d->chunk, dt, A, la2, gpre, s);
    if (e != cudaSuccess) return cuda_fail(e, "dart_sma_forward_decayed: decay terms");
    dart::SmaArgs a{d->batch, d->seqlen, d->nheads, d->headdim, d->dstate, d->chunk, d->ngroups,
                    Q, E, Cm, dH, g, y_ssd, out, status_word(), la2, gpre};
    if (!a.status) return fail(DART_ERR_CUDA, "dart_sma_forward_decayed: no device status word");
    e = dart::launch_sma(a, dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "dart_sma_forward_decayed launch");
    return DART_OK;
}

size_t dart_ssd_scan_backward_workspace_bytes(const dart_dims* d) {
    if (!d) return 0;
    return dart::scan_bwd_workspace_bytes(d->batch, d->seqlen, d->nheads, d->dstate, d->headdim, d->chunk);
}

dart_status dart_ssd_scan_backward(const dart_dims* d, dart_dtype dtype, const void* x, const float* dt,
                                   const float* A, const void* Bm, const void* Cm, const float* init_state,
                                   const float* states, const float* dy, const float* ddH, const float* dCm_add,
                                   float* dx, float* ddt, float* dA, float* dBm, float* dCm, float* dinit_state,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    t_err[0] = 0;
    dart_status st = check_common(d, dtype, true);
    if (st != DART_OK) return st;
    if (!dart::scan_bwd_supported(d->dstate, d->headdim, d->chunk))
        return fail(DART_ERR_UNSUPPORTED, "dart_ssd_scan_backward: (N=%d, P=%d, S=%d) not compiled", d->dstate,
                    d->headdim, d->chunk);
    DART_REQUIRE_PTR(x); DART_REQUIRE_PTR(dt); DART_REQUIRE_PTR(A); DART_REQUIRE_PTR(Bm); DART_REQUIRE_PTR(Cm);
    DART_OPTIONAL_PTR(init_state); DART_REQUIRE_PTR(states); DART_REQUIRE_PTR(dy); DART_OPTIONAL_PTR(ddH);
    DART_OPTIONAL_PTR(dCm_add); DART_REQUIRE_PTR(dx); DART_REQUIRE_PTR(ddt); DART_REQUIRE_PTR(dA); DART_REQUIRE_PTR(dBm); DART_REQUIRE_PTR(dCm);
    DART_OPTIONAL_PTR(dinit_state); DART_REQUIRE_PTR(workspace);
    const size_t need = dart_ssd_scan_backward_workspace_bytes(d);
    if (workspace_bytes < need)
        return fail(DART_ERR_INVALID_ARG, "workspace: %zu bytes, need %zu", workspace_bytes, need);
    dart::ScanBwdArgs a{d->batch, d->seqlen, d->nheads, d->headdim, d->dstate, d->chunk, d->ngroups, x, dt, A, Bm, Cm,
                        init_state, states, dy, ddH, dCm_add, dx, ddt, dA, dBm, dCm, dinit_state, status_word()};
    if (!a.status) return fail(DART_ERR_CUDA, "dart_ssd_scan_backward: no device status word");
    cudaError_t e = dart::launch_ssd_scan_bwd(a, workspace, dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dart_ssd_scan_backward launch");
    return DART_OK;
}

size_t dart_sma_backward_workspace_bytes(const dart_dims* d) {
    if (!d) return 0;
    return dart::sma_bwd_workspace_bytes(d->batch, d->seqlen, d->nheads, d->dstate, d->chunk);
}

dart_status dart_sma_backward(const dart_dims* d, dart_dtype dtype, const void* Q, const void* E, const void* Cm,
                              const void* dH, float g, const float* dy, float* dQ, float* dE, float* dCm,
                              float* ddH, float* dg, void* workspace, size_t workspace_bytes, void* stream) {
    t_err[0] = 0;
    dart_status st = check_common(d, dtype, true);
    if (st != DART_OK) return st;
    if (!dart::sma_supported(d->dstate, d->headdim, d->chunk, dtype))
        return fail(DART_ERR_UNSUPPORTED, "dart_sma_backward: (N=%d, P=%d, S=%d) not compiled", d->dstate,
                    d->headdim, d->chunk);
    DART_REQUIRE_PTR(Q); DART_REQUIRE_PTR(E); DART_REQUIRE_PTR(Cm); DART_REQUIRE_PTR(dH); DART_REQUIRE_PTR(dy);
    DART_REQUIRE_PTR(dQ); DART_REQUIRE_PTR(dE); DART_REQUIRE_PTR(dCm); DART_REQUIRE_PTR(ddH); DART_REQUIRE_PTR(dg);
    DART_REQUIRE_PTR(workspace);
    const size_t need = dart_sma_backward_workspace_bytes(d);
    if (workspace_bytes < need)
        return fail(DART_ERR_INVALID_ARG, "workspace: %zu bytes, need %zu", workspace_bytes, need);
    dart::SmaBwdArgs a{d->batch, d->seqlen, d->nheads, d->headdim, d->dstate, d->chunk, d->ngroups, Q, E, Cm, dH, g, dy,
                       dQ, dE, dCm, ddH, dg, status_word()};
    if (!a.status) return fail(DART_ERR_CUDA, "dart_sma_backward: no device status word");
    cudaError_t e = dart::launch_sma_bwd(a, workspace, dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dart_sma_backward launch");
    return DART_OK;
}

size_t dart_decode_step_workspace_bytes(const dart_dims* d, dart_dtype, int cmax) {
    if (!d || cmax < 0 || cmax > dart::kDecodeMaxCmax) return 0;
    const size_t ns = (size_t)dart::decode_num_splits(d->batch, d->nheads, cmax);
    return sizeof(float) * (size_t)d->batch * (size_t)d->nheads * ns * (2 + 2 * (size_t)d->headdim);
}

dart_status dart_decode_step(const dart_dims* d, dart_dtype dtype, const void* x_t, const float* dt_t,
                             const float* A, const void* B_t, const void* C_t, const void* Q_t,
                             const void* E_t, float g, float* state, float* dH_cur, void* dH_cache,
                             int cmax, int* n_chunks, int* pos, float* y, void* workspace,
                             size_t workspace_bytes, void* stream) {
    t_err[0] = 0;
    dart_status st = check_common(d, dtype, false);
    if (st != DART_OK) return st;
    if (!dart::decode_supported(d->dstate, d->headdim, d->chunk, dtype))
        return fail(DART_ERR_UNSUPPORTED, "dart_decode_step: (N=%d, P=%d) not compiled", d->dstate, d->headdim);
    if (cmax < 1 || cmax > dart::kDecodeMaxCmax)
        return fail(DART_ERR_INVALID_ARG, "cmax = %d outside [1, %d]", cmax, dart::kDecodeMaxCmax);
    DART_REQUIRE_PTR(x_t); DART_REQUIRE_PTR(dt_t); DART_REQUIRE_PTR(A); DART_REQUIRE_PTR(B_t);
    DART_REQUIRE_PTR(C_t); DART_REQUIRE_PTR(Q_t); DART_REQUIRE_PTR(E_t); DART_REQUIRE_PTR(state);
    DART_REQUIRE_PTR(dH_cur); DART_REQUIRE_PTR(dH_cache); DART_REQUIRE_PTR(n_chunks);
    DART_REQUIRE_PTR(pos); DART_REQUIRE_PTR(y); DART_REQUIRE_PTR(workspace);
    if (workspace_bytes < dart_decode_step_workspace_bytes(d, dtype, cmax))
        return fail(DART_ERR_INVALID_ARG, "workspace: %zu bytes, need %zu", workspace_bytes,
                    dart_decode_step_workspace_bytes(d, dtype, cmax));
    dart::DecodeArgs a{d->batch, d->nheads, d->headdim, d->dstate, d->chunk, d->ngroups, cmax,
                       dart::decode_num_splits(d->batch, d->nheads, cmax),
                       x_t, dt_t, A, B_t, C_t, Q_t, E_t, g, state, dH_cur, dH_cache,
                       n_chunks, pos, y, static_cast<float*>(workspace), status_word()};
    if (!a.status) return fail(DART_ERR_CUDA, "dart_decode_step: no device status word");
    cudaError_t e = dart::launch_decode(a, dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dart_decode_step launch");
    return DART_OK;
}

dart_status dart_decode_step_decayed(const dart_dims* d, dart_dtype dtype, const void* x_t, const float* dt_t,
                                     const float* A, const void* B_t, const void* C_t, const void* Q_t,
                                     const void* E_t, float g, float* state, float* dH_cur, void* dH_cache,
                                     int cmax, int* n_chunks, int* pos, float* mem_logdecay, float* y,
                                     void* workspace, size_t workspace_bytes, void* stream) {
    t_err[0] = 0;
    dart_status st = check_common(d, dtype, false);
    if (st != DART_OK) return st;
    if (!dart::decode_supported(d->dstate, d->headdim, d->chunk, dtype))
        return fail(DART_ERR_UNSUPPORTED, "dart_decode_step_decayed: (N=%d, P=%d) not compiled", d->dstate,
                    d->headdim);
    if (cmax < 1 || cmax > dart::kDecodeMaxCmax)
        return fail(DART_ERR_INVALID_ARG, "cmax = %d outside [1, %d]", cmax, dart::kDecodeMaxCmax);
    DART_REQUIRE_PTR(x_t); DART_REQUIRE_PTR(dt_t); DART_REQUIRE_PTR(A); DART_REQUIRE_PTR(B_t);
    DART_REQUIRE_PTR(C_t); DART_REQUIRE_PTR(Q_t); DART_REQUIRE_PTR(E_t); DART_REQUIRE_PTR(state);
    DART_REQUIRE_PTR(dH_cur); DART_REQUIRE_PTR(dH_cache); DART_REQUIRE_PTR(n_chunks);
    DART_REQUIRE_PTR(pos); DART_REQUIRE_PTR(mem_logdecay); DART_REQUIRE_PTR(y); DART_REQUIRE_PTR(workspace);
    if (workspace_bytes < dart_decode_step_workspace_bytes(d, dtype, cmax))
        return fail(DART_ERR_INVALID_ARG, "workspace: %zu bytes, need %zu", workspace_bytes,
                    dart_decode_step_workspace_bytes(d, dtype, cmax));
    dart::DecodeArgs a{d->batch, d->nheads, d->headdim, d->dstate, d->chunk, d->ngroups, cmax,
                       dart::decode_num_splits(d->batch, d->nheads, cmax),
                       x_t, dt_t, A, B_t, C_t, Q_t, E_t, g, state, dH_cur, dH_cache,
                       n_chunks, pos, y, static_cast<float*>(workspace), status_word(), mem_logdecay};
    if (!a.status) return fail(DART_ERR_CUDA, "dart_decode_step_decayed: no device status word");
    cudaError_t e = dart::launch_decode(a, dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dart_decode_step_decayed launch");
    return DART_OK;
}

dart_status dart_decode_step_e4m3(const dart_dims* d, dart_dtype dtype, const void* x_t, const float* dt_t,
                                  const float* A, const void* B_t, const void* C_t, const void* Q_t,
                                  const void* E_t, float g, float* state, float* dH_cur, unsigned char* cache,
                                  signed char* cache_exp, int cmax, int* n_chunks, int* pos, float* mem_logdecay,
                                  float* y, void* workspace, size_t workspace_bytes, void* stream) {
    t_err[0] = 0;
    dart_status st = check_common(d, dtype, false);
    if (st != DART_OK) return st;
    if (!dart::decode_e4m3_supported(d->dstate, d->headdim))
        return fail(DART_ERR_UNSUPPORTED, "dart_decode_step_e4m3: (N=%d, P=%d) not compiled (P = 64, N = 64 or 128)",
                    d->dstate, d->headdim);
    if (cmax < 1 || cmax > dart::kDecodeMaxCmax)
        return fail(DART_ERR_INVALID_ARG, "cmax = %d outside [1, %d]", cmax, dart::kDecodeMaxCmax);
    DART_REQUIRE_PTR(x_t); DART_REQUIRE_PTR(dt_t); DART_REQUIRE_PTR(A); DART_REQUIRE_PTR(B_t);
    DART_REQUIRE_PTR(C_t); DART_REQUIRE_PTR(Q_t); DART_REQUIRE_PTR(E_t); DART_REQUIRE_PTR(state);
    DART_REQUIRE_PTR(dH_cur); DART_REQUIRE_PTR(cache); DART_REQUIRE_PTR(cache_exp); DART_REQUIRE_PTR(n_chunks);
    DART_REQUIRE_PTR(pos); DART_OPTIONAL_PTR(mem_logdecay); DART_REQUIRE_PTR(y); DART_REQUIRE_PTR(workspace);
    if (workspace_bytes < dart_decode_step_workspace_bytes(d, dtype, cmax))
        return fail(DART_ERR_INVALID_ARG, "workspace: %zu bytes, need %zu", workspace_bytes,
                    dart_decode_step_workspace_bytes(d, dtype, cmax));
    dart::DecodeArgs a{d->batch, d->nheads, d->headdim, d->dstate, d->chunk, d->ngroups, cmax,
                       dart::decode_num_splits(d->batch, d->nheads, cmax),
                       x_t, dt_t, A, B_t, C_t, Q_t, E_t, g, state, dH_cur, cache,
                       n_chunks, pos, y, static_cast<float*>(workspace), status_word(), mem_logdecay, cache_exp};
    if (!a.status) return fail(DART_ERR_CUDA, "dart_decode_step_e4m3: no device status word");
    cudaError_t e = dart::launch_decode_e4m3(a, dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dart_decode_step_e4m3 launch");
    return DART_OK;
}

dart_status dart_cache_quantize_e4m3(const dart_dims* d, dart_dtype dtype, const void* dH, int nmem,
                                     unsigned char* cache, signed char* cache_exp, int cmax, void* stream) {
    t_err[0] = 0;
    dart_status st = check_common(d, dtype, true);
    if (st != DART_OK) return st;
    if (!dart::decode_e4m3_supported(d->dstate, d->headdim))
        return fail(DART_ERR_UNSUPPORTED, "dart_cache_quantize_e4m3: (N=%d, P=%d) not compiled", d->dstate,
                    d->headdim);
    const int C = (d->seqlen + d->chunk - 1) / d->chunk;
    if (nmem < 0 || nmem > C || nmem > cmax)
        return fail(DART_ERR_INVALID_ARG, "dart_cache_quantize_e4m3: nmem = %d outside [0, min(C = %d, cmax = %d)]",
                    nmem, C, cmax);
    DART_REQUIRE_PTR(dH); DART_REQUIRE_PTR(cache); DART_REQUIRE_PTR(cache_exp);
    cudaError_t e = dart::launch_cache_quantize_e4m3(d->batch, d->nheads, C, d->dstate, d->headdim, nmem, cmax, dH,
                                                     dtype, cache, cache_exp, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dart_cache_quantize_e4m3 launch");
    return DART_OK;
}

dart_status dart_decode_memlog_init(const dart_dims* d, const float* dt, const float* A, float* mem_logdecay,
                                    int cmax, void* stream) {
    t_err[0] = 0;
    if (!d) return fail(DART_ERR_INVALID_ARG, "dims is NULL");
    if (d->batch < 1 || d->seqlen < 1 || d->nheads < 1 || d->chunk < 1)
        return fail(DART_ERR_INVALID_ARG, "dart_decode_memlog_init: batch, seqlen, nheads and chunk must be >= 1");
    if (cmax < 1 || d->seqlen / d->chunk > cmax)
        return fail(DART_ERR_INVALID_ARG, "dart_decode_memlog_init: %d completed chunks do not fit cmax = %d",
                    d->seqlen / d->chunk, cmax);
    DART_REQUIRE_PTR(dt); DART_REQUIRE_PTR(A); DART_REQUIRE_PTR(mem_logdecay);
    cudaError_t e = dart::launch_decode_memlog_init(d->batch, d->seqlen, d->nheads, d->chunk, cmax, dt, A,
                                                    mem_logdecay, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dart_decode_memlog_init launch");
    return DART_OK;
}

// The decode step for callers that cannot allocate device memory: the split
// partials go to the library's fixed static scratch (decode.cu) instead of a
// caller workspace.  Validation matches dart_decode_step, plus the scratch
// size limit; no allocation of any kind happens here.
dart_status dart_decode_step_noalloc(const dart_dims* d, dart_dtype dtype, const void* x_t, const float* dt_t,
                                     const float* A, const void* B_t, const void* C_t, const void* Q_t,
                                     const void* E_t, float g, float* state, float* dH_cur, void* dH_cache,
                                     int cmax, int* n_chunks, int* pos, float* y, void* stream) {
    t_err[0] = 0;
    dart_status st = check_common(d, dtype, false);
    if (st != DART_OK) return st;
    if (!dart::decode_supported(d->dstate, d->headdim, d->chunk, dtype))
        return fail(DART_ERR_UNSUPPORTED, "dart_decode_step_noalloc: (N=%d, P=%d) not compiled", d->dstate,
                    d->headdim);
    if (cmax < 1 || cmax > dart::kDecodeMaxCmax)
        return fail(DART_ERR_INVALID_ARG, "cmax = %d outside [1, %d]", cmax, dart::kDecodeMaxCmax);
    DART_REQUIRE_PTR(x_t); DART_REQUIRE_PTR(dt_t); DART_REQUIRE_PTR(A); DART_REQUIRE_PTR(B_t);
    DART_REQUIRE_PTR(C_t); DART_REQUIRE_PTR(Q_t); DART_REQUIRE_PTR(E_t); DART_REQUIRE_PTR(state);
    DART_REQUIRE_PTR(dH_cur); DART_REQUIRE_PTR(dH_cache); DART_REQUIRE_PTR(n_chunks);
    DART_REQUIRE_PTR(pos); DART_REQUIRE_PTR(y);
    const size_t need = dart_decode_step_workspace_bytes(d, dtype, cmax);
    if (need > dart::kNoAllocScratchBytes)
        return fail(DART_ERR_UNSUPPORTED,
                    "dart_decode_step_noalloc: this batch needs %zu bytes of scratch, more than the fixed %zu; "
                    "use dart_decode_step with a workspace or fewer sequences / a smaller cmax",
                    need, dart::kNoAllocScratchBytes);
    void* scratch = nullptr;
    cudaError_t e = dart::noalloc_scratch(&scratch);
    if (e != cudaSuccess) return cuda_fail(e, "dart_decode_step_noalloc: static scratch address");
    dart::DecodeArgs a{d->batch, d->nheads, d->headdim, d->dstate, d->chunk, d->ngroups, cmax,
                       dart::decode_num_splits(d->batch, d->nheads, cmax),
                       x_t, dt_t, A, B_t, C_t, Q_t, E_t, g, state, dH_cur, dH_cache,
                       n_chunks, pos, y, static_cast<float*>(scratch), status_word()};
    if (!a.status) return fail(DART_ERR_CUDA, "dart_decode_step_noalloc: no device status word");
    e = dart::launch_decode(a, dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dart_decode_step_noalloc launch");
    return DART_OK;
}

dart_status dart_selftest_wait_timeout(unsigned int limit_us, void* stream) {
    t_err[0] = 0;
    if (limit_us < 1 || limit_us > 2000000)
        return fail(DART_ERR_INVALID_ARG, "dart_selftest_wait_timeout: limit_us = %u outside [1, 2000000]", limit_us);
    int* status = status_word();
    if (!status) return fail(DART_ERR_CUDA, "dart_selftest_wait_timeout: no device status word");
    cudaError_t e = dart::launch_wait_drill(status, 1000ull * limit_us, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dart_selftest_wait_timeout launch");
    dart::count_launches(1);
    return DART_OK;
}

dart_status dart_sync_status(void* stream) {
    t_err[0] = 0;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dart_sync_status: stream synchronize");
    int words[2] = {0, 0};
    e = cudaMemcpyFromSymbol(words, dart::g_status, sizeof(words));
    if (e != cudaSuccess) return cuda_fail(e, "dart_sync_status: read status");
    if (words[0] || words[1]) {
        const int zero[2] = {0, 0};
        e = cudaMemcpyToSymbol(dart::g_status, zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "dart_sync_status: clear status");
    }
    if (words[0] & dart::kStatusTimeout)
        return fail(DART_ERR_TIMEOUT, "a bounded device wait gave up (kernel %d, wait site %d)", words[1] >> 8,
                    words[1] & 0xff);
    if (words[0] & dart::kStatusDevice)
        return fail(DART_ERR_DEVICE, "device flagged bad state (decode counters out of range or cache full)");
    return DART_OK;
}

}  // extern "C"
