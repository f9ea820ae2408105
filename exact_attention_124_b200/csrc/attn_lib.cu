// attn_lib.cu -- the C ABI (include/attn.h, include/attn_selftest.h): argument
// checks, TMA tensor maps, launches.  The whole library is this one
// translation unit, so the device status word has a single definition.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>

#include "attn.h"
#include "attn_selftest.h"
#include "backward.cuh"
#include "decode.cuh"
#include "fused_fwd.cuh"
#include "selftest.cuh"
#include "unfused.cuh"

namespace {

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per barrier wait
constexpr int kMaxDevices = 64;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
int g_mma_order = 0;
int g_exp_split = -1;  // pairs of every 8 on the FMA pipe; -1: per-head-size default
constexpr int kDefaultSplit64 = 0, kDefaultSplit128 = 0;  // measured fastest on B200
unsigned int g_last_where = 0;

// Per-device state is tied to the CUDA context it was set up in: kernel
// attributes, the library's streams and events and the static workspace's
// device address all die with the context (cudaDeviceReset, or any teardown
// of the primary context), so every entry point compares the current
// context's process-unique id with the recorded one and sets up again on a
// mismatch.  Handles of a destroyed context are dropped, never used.
struct DeviceState {
    bool ready = false;
    unsigned long long ctx_id = 0;
    int sms = 0;
    void *noalloc_ws = nullptr;  // device address of the static workspace, looked up once
};
DeviceState g_dev[kMaxDevices];

using PfnCtxGetCurrent = CUresult (*)(CUcontext *);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long *);
PfnCtxGetCurrent g_ctx_get_current = nullptr;
PfnCtxGetId g_ctx_get_id = nullptr;

template <typename F>
bool driver_fn(const char *name, F &out)
{
    if (out) return true;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr) {
        (void)cudaGetLastError();
        return false;
    }
    out = reinterpret_cast<F>(fn);
    return true;
}

// Process-unique id of the current device's context (creating the primary
// context if none is current yet); 0 on failure.  Makes no runtime call while
// a context is current, so the entry points can be captured into a CUDA graph
// (stream capture forbids cudaFree, the usual way to bind the context).
unsigned long long current_ctx_id()
{
    if (!driver_fn("cuCtxGetCurrent", g_ctx_get_current) || !driver_fn("cuCtxGetId", g_ctx_get_id))
        return 0;
    CUcontext ctx = nullptr;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return 0;
    if (ctx == nullptr) {
        // no context on this thread yet (never the case during a capture):
        // make the runtime bind its primary context
        if (cudaFree(nullptr) != cudaSuccess) {
            (void)cudaGetLastError();
            return 0;
        }
        if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    }
    unsigned long long id = 0;
    if (g_ctx_get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// attn_fwd_host's copy pipeline: two non-blocking streams (host -> device,
// device -> host) and events per chunk, created on first use per device.
constexpr int kHostChunks = 8;
struct HostPipe {
    bool ready = false;
    unsigned long long ctx_id = 0;
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t loaded[kHostChunks] = {}, computed[kHostChunks] = {};
};
HostPipe g_pipe[kMaxDevices];

// Called after device_ready(), which has checked the device and context.
HostPipe *host_pipe()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    HostPipe &hp = g_pipe[dev];
    if (hp.ready && hp.ctx_id == g_dev[dev].ctx_id) return &hp;
    hp = HostPipe{};  // a previous context's handles are gone with it
    bool ok = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.done, cudaEventDisableTiming) == cudaSuccess;
    for (int c = 0; ok && c < kHostChunks; ++c)
        ok = cudaEventCreateWithFlags(&hp.loaded[c], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&hp.computed[c], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        (void)cudaGetLastError();
        return nullptr;
    }
    hp.ctx_id = g_dev[dev].ctx_id;
    hp.ready = true;
    return &hp;
}

int get_encoder()
{
    if (g_encode) return ATTN_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr) {
        (void)cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return ATTN_OK;
}

template <typename K>
bool set_smem(K kernel, int bytes)
{
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
           cudaSuccess;
}

// The fused kernel re-balances registers with setmaxnreg; an increase that
// the launch's registers cannot cover would wait forever, so refuse to launch
// a build whose per-thread register count is below the split's assumption.
template <int D, int EMU, bool CAUSAL>
bool fused_ready1()
{
    using C = attn::FusedCfg<D>;
    if (!set_smem(attn::attn_fwd_fused_kernel<D, EMU, CAUSAL>, CAUSAL ? C::SMEM : C::SMEM_NC)) return false;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, attn::attn_fwd_fused_kernel<D, EMU, CAUSAL>) != cudaSuccess)
        return false;
    return fa.numRegs >= C::REGS_LAUNCH && fa.maxThreadsPerBlock >= C::THREADS;
}

template <int D, int EMU>
bool fused_ready()
{
    return fused_ready1<D, EMU, true>() && fused_ready1<D, EMU, false>();
}

template <int D>
bool fused_all_ready()
{
    return fused_ready<D, 0>() && fused_ready<D, 2>() && fused_ready<D, 3>() &&
           fused_ready<D, 4>();
}

// Per-device, per-context set-up: device check (compute capability 10.0),
// SM count, shared-memory opt-in of every kernel.  Runs again when the
// device's context has changed since the last set-up.
int device_ready(int *sms_out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        (void)cudaGetLastError();
        return ATTN_ERR_NO_DEVICE;
    }
    const unsigned long long ctx = current_ctx_id();
    if (ctx == 0) return ATTN_ERR_NO_DEVICE;
    DeviceState &st = g_dev[dev];
    if (!st.ready || st.ctx_id != ctx) {
        st = DeviceState{};
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            (void)cudaGetLastError();
            return ATTN_ERR_NO_DEVICE;
        }
        if (major != 10 || minor != 0 || sms < 1) return ATTN_ERR_NO_DEVICE;
        if (get_encoder() != ATTN_OK) return ATTN_ERR_LAUNCH;
        bool ok = true;
        ok &= set_smem(attn::bwd_dkdv64_kernel, attn::Dkdv64Cfg::SMEM);
        ok &= set_smem(attn::bwd_dkdv_kernel<128>, attn::BwdCfg<128>::SMEM);
        ok &= set_smem(attn::bwd_dq_kernel<64>, attn::DqCfg<64>::SMEM);
        ok &= set_smem(attn::bwd_dq_kernel<128>, attn::DqCfg<128>::SMEM);
        ok &= set_smem(attn::decode_partial_kernel<64, 1>, attn::DecCfg<64>::SMEM);
        ok &= set_smem(attn::decode_partial_kernel<64, 2>, attn::DecCfg<64>::SMEM);
        ok &= set_smem(attn::decode_partial_kernel<64, 4>, attn::DecCfg<64>::SMEM);
        ok &= set_smem(attn::decode_partial_kernel<128, 1>, attn::DecCfg<128>::SMEM);
        ok &= set_smem(attn::decode_partial_kernel<128, 2>, attn::DecCfg<128>::SMEM);
        ok &= set_smem(attn::decode_partial_kernel<128, 4>, attn::DecCfg<128>::SMEM);
        ok &= fused_all_ready<64>();
        ok &= fused_all_ready<128>();
        ok &= set_smem(attn::s_gemm_kernel<64>, attn::K1Cfg<64>::SMEM);
        ok &= set_smem(attn::s_gemm_kernel<128>, attn::K1Cfg<128>::SMEM);
        ok &= set_smem(attn::pv_gemm_kernel<64>, attn::PvCfg<64>::SMEM);
        ok &= set_smem(attn::pv_gemm_kernel<128>, attn::PvCfg<128>::SMEM);
        ok &= set_smem(attn::selftest_qk_kernel<64>, 1024 + 2 * 128 * 64 * 2 + 64);
        ok &= set_smem(attn::selftest_qk_kernel<128>, 1024 + 2 * 128 * 128 * 2 + 64);
        ok &= set_smem(attn::selftest_pv_kernel<64>, 1024 + 128 * 64 * 2 + 64);
        ok &= set_smem(attn::selftest_pv_kernel<128>, 1024 + 128 * 128 * 2 + 64);
        if (!ok) {
            (void)cudaGetLastError();
            return ATTN_ERR_LAUNCH;
        }
        st.sms = sms;
        st.ctx_id = ctx;
        st.ready = true;
    }
    if (sms_out) *sms_out = st.sms;
    return ATTN_OK;
}

// bf16 tensor [heads, rows, inner] as a 3-D TMA map with 128-byte swizzle and
// a box of (64, box_rows, 1) elements; out-of-range rows read as zero.
int make_map(CUtensorMap *m, const void *ptr, uint64_t inner, uint64_t rows, uint64_t heads,
             uint32_t box_rows)
{
    cuuint64_t dims[3] = {inner, rows, heads};
    cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_LAUNCH;
}

bool misaligned(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }
// lse is read and written one float at a time: 4-byte alignment suffices.
bool misaligned_f32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) != 0; }

// Host-side checks shared by every forward entry point; no CUDA call here.
int validate(const void *q, const void *k, const void *v, const void *o, const void *lse, int B,
             int H, int T, int d_h, int causal, float scale)
{
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
    if (d_h != 64 && d_h != 128) return ATTN_ERR_UNSUPPORTED_DH;
    if (B < 1 || H < 1 || T < 1) return ATTN_ERR_BAD_SHAPE;
    const long long bh = (long long)B * H;
    if (bh * (long long)T > (long long)INT_MAX || T > INT_MAX - 256) return ATTN_ERR_BAD_SHAPE;
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(o) || misaligned_f32(lse))
        return ATTN_ERR_ALIGN;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_BAD_SCALE;
    if (causal != 0 && causal != 1) return ATTN_ERR_BAD_ARG;
    return ATTN_OK;
}

int launch_status()
{
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

// Persistent grid: one CTA per SM, or fewer when there is less work (causal
// work is dealt in pairs of query blocks, non-causal in single blocks).
int fused_grid(long long BH, int T, int causal, int sms)
{
    const long long nqb = (T + 255) / 256;
    const long long work = causal ? BH * ((nqb + 1) / 2) : BH * nqb;
    return (int)(work < sms ? work : sms);
}

// Kernel parameters of a fused launch (output pointers left null).
attn::FusedParams fused_params(int B, int H, int H_kv, int T, int causal, float scale)
{
    attn::FusedParams p;
    p.o = nullptr;
    p.lse = nullptr;
    p.BH = B * H;
    p.H = H;
    p.group = H / H_kv;
    p.T = T;
    p.causal = causal;
    p.c_log2 = scale * 1.4426950408889634f;
    p.nqb = (T + 255) / 256;
    p.units = p.BH * p.nqb;
    p.nkv = (T + 127) / 128;
    p.order_mode = g_mma_order;
    p.limit_ns = kWaitLimitNs;
    return p;
}

template <int D>
int launch_fused(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
                 int H_kv, int T, int causal, float scale, cudaStream_t stream, int sms)
{
    using C = attn::FusedCfg<D>;
    const int BH = B * H;
    CUtensorMap mq, mk, mv;
    if (make_map(&mq, q, D, T, BH, 128) || make_map(&mk, k, D, T, (uint64_t)B * H_kv, 128) ||
        make_map(&mv, v, D, T, (uint64_t)B * H_kv, 128))
        return ATTN_ERR_LAUNCH;
    attn::FusedParams p = fused_params(B, H, H_kv, T, causal, scale);
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    const int grid = fused_grid(BH, T, causal, sms);
    const int split = g_exp_split >= 0 ? g_exp_split : (D == 64 ? kDefaultSplit64 : kDefaultSplit128);
    // One kernel instance per mask mode.  The causal one stores each thread's O
    // row straight to global memory; the non-causal one passes a warp's rows
    // through shared memory (whole 128-byte lines per store) and needs the
    // larger shared-memory size.  The causal kernel is faster with the direct
    // stores: its epilogue timing keeps the two warpgroups out of step.
    if (causal) {
        switch (split) {
            case 0: attn::attn_fwd_fused_kernel<D, 0, true><<<grid, C::THREADS, C::SMEM, stream>>>(mq, mk, mv, p); break;
            case 2: attn::attn_fwd_fused_kernel<D, 2, true><<<grid, C::THREADS, C::SMEM, stream>>>(mq, mk, mv, p); break;
            case 3: attn::attn_fwd_fused_kernel<D, 3, true><<<grid, C::THREADS, C::SMEM, stream>>>(mq, mk, mv, p); break;
            default: attn::attn_fwd_fused_kernel<D, 4, true><<<grid, C::THREADS, C::SMEM, stream>>>(mq, mk, mv, p); break;
        }
    } else {
        switch (split) {
            case 0: attn::attn_fwd_fused_kernel<D, 0, false><<<grid, C::THREADS, C::SMEM_NC, stream>>>(mq, mk, mv, p); break;
            case 2: attn::attn_fwd_fused_kernel<D, 2, false><<<grid, C::THREADS, C::SMEM_NC, stream>>>(mq, mk, mv, p); break;
            case 3: attn::attn_fwd_fused_kernel<D, 3, false><<<grid, C::THREADS, C::SMEM_NC, stream>>>(mq, mk, mv, p); break;
            default: attn::attn_fwd_fused_kernel<D, 4, false><<<grid, C::THREADS, C::SMEM_NC, stream>>>(mq, mk, mv, p); break;
        }
    }
    return launch_status();
}

template <int D>
int launch_unfused(const void *q, const void *k, const void *v, void *o, float *lse, void *s_ws,
                   void *p_ws, int BH, int T, int causal, float scale, cudaStream_t stream, int sms)
{
    CUtensorMap mq, mk, ms, mp, mv;
    if (make_map(&mq, q, D, T, BH, 128) || make_map(&mk, k, D, T, BH, 128) ||
        make_map(&ms, s_ws, T, T, BH, 128) || make_map(&mp, p_ws, T, T, BH, 128) ||
        make_map(&mv, v, D, T, BH, 64))
        return ATTN_ERR_LAUNCH;
    attn::UnfusedParams p;
    p.BH = BH;
    p.T = T;
    p.causal = causal;
    p.c_log2 = scale * 1.4426950408889634f;
    p.limit_ns = kWaitLimitNs;
    auto *S = static_cast<__nv_bfloat16 *>(s_ws);
    auto *P = static_cast<__nv_bfloat16 *>(p_ws);
    {  // persistent: one CTA per SM over the tiles of S (under the causal mask, the lower ones)
        const long long nt = T / 128;
        const long long tiles = (causal ? nt * (nt + 1) / 2 : nt * nt) * BH;
        const int grid = (int)(tiles < sms ? tiles : sms);
        attn::s_gemm_kernel<D><<<grid, attn::K1Cfg<D>::THREADS, attn::K1Cfg<D>::SMEM, stream>>>(mq, mk, ms, p);
    }
    if (launch_status()) return ATTN_ERR_LAUNCH;
    const long long rows = (long long)BH * T;
    attn::softmax_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(S, P, lse, p);
    if (launch_status()) return ATTN_ERR_LAUNCH;
    attn::pv_gemm_kernel<D><<<dim3(T / 128, BH), 128, attn::PvCfg<D>::SMEM, stream>>>(
        mp, mv, static_cast<__nv_bfloat16 *>(o), p);
    return launch_status();
}

template <int D>
int launch_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
               const void *dout, void *dq, void *dk, void *dv, void *ws, int B, int H, int H_kv,
               int T, int causal, float scale, cudaStream_t stream)
{
    using C = attn::BwdCfg<D>;
    const int BH = B * H, BHkv = B * H_kv;
    CUtensorMap mq, mk, mv, mg;
    if (make_map(&mq, q, D, T, BH, 128) || make_map(&mg, dout, D, T, BH, 128) ||
        make_map(&mk, k, D, T, BHkv, 128) || make_map(&mv, v, D, T, BHkv, 128))
        return ATTN_ERR_LAUNCH;
    auto *stats = static_cast<float2 *>(ws);
    const int nq = (T + 127) / 128, Tp = 128 * nq;  // a ragged last block is padded
    const long long prow = (long long)BH * Tp;
    attn::bwd_stats_kernel<D><<<(unsigned)((prow + 7) / 8), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(dout), lse,
        stats, prow, T, Tp);
    if (launch_status()) return ATTN_ERR_LAUNCH;
    attn::BwdParams p;
    p.stats = stats;
    p.H = H;
    p.H_kv = H_kv;
    p.group = H / H_kv;
    p.T = T;
    p.nq = nq;
    p.Tp = Tp;
    p.causal = causal;
    p.c_log2 = scale * 1.4426950408889634f;
    p.scale = scale;
    p.limit_ns = kWaitLimitNs;
    p.out_a = static_cast<__nv_bfloat16 *>(dk);
    p.out_b = static_cast<__nv_bfloat16 *>(dv);
    if constexpr (D == 64)  // room for 128-wide score MMAs and two S^T buffers at d_h = 64
        attn::bwd_dkdv64_kernel<<<dim3(nq, BHkv), attn::Dkdv64Cfg::THREADS, attn::Dkdv64Cfg::SMEM,
                                  stream>>>(mq, mk, mv, mg, p);
    else
        attn::bwd_dkdv_kernel<D><<<dim3(nq, BHkv), C::THREADS, C::SMEM, stream>>>(mq, mk, mv, mg, p);
    if (launch_status()) return ATTN_ERR_LAUNCH;
    p.out_a = static_cast<__nv_bfloat16 *>(dq);
    p.out_b = nullptr;
    using Q = attn::DqCfg<D>;
    attn::bwd_dq_kernel<D><<<dim3(nq, BH), Q::THREADS, Q::SMEM, stream>>>(mq, mk, mv, mg, p);
    return launch_status();
}

// Work plan of the decode path (see decode_geometry).
struct DecGeom {
    int nkt, nrb, balanced, chunk, eff, G, slots;
    int copies;  // copies of the packed rows in the 128-row tile (4, 2 or 1)
    long long tot;
};

// splits > 0: every head cut into `splits` key ranges (clamped to the tile
// count), one CTA each.  splits < 0: balanced ranges of the (head, key tile)
// list, one CTA per SM.  splits == 0: the fixed split that fills one wave of
// CTAs (one per SM) if that keeps at least 85 % of the SMs busy -- no range
// boundary inside a CTA, no second wave -- else balanced.
void decode_geometry(int B, int H, int H_kv, int Tq, int Tk, int splits, int sms, DecGeom &g)
{
    g.nkt = (Tk + 127) / 128;
    const long long rows = (long long)(H / H_kv) * Tq;  // packed rows per K/V head
    g.copies = rows <= 32 ? 4 : rows <= 64 ? 2 : 1;
    g.nrb = (int)((rows + 127) / 128);
    g.tot = (long long)B * H_kv * g.nrb * g.nkt;
    const long long heads = (long long)B * H_kv * g.nrb;
    if (splits == 0) {
        const long long s = std::min<long long>(sms / heads, g.nkt);
        const long long chunk = s > 0 ? (g.nkt + s - 1) / s : 0;
        const long long busy = s > 0 ? heads * ((g.nkt + chunk - 1) / chunk) : 0;
        splits = (s > 0 && 100 * busy >= 85LL * sms) ? (int)s : -1;
    }
    if (splits < 0) {
        g.balanced = 1;
        g.G = (int)std::min<long long>(sms, g.tot);
        const long long per = g.tot / g.G;  // tiles per CTA, rounded down (>= 1)
        // a head's nkt consecutive tiles meet at most (nkt - 1) / per + 2 ranges
        g.slots = (int)std::min<long long>(g.G, (g.nkt - 1) / per + 2);
        g.chunk = 0;
        g.eff = 0;
    } else {
        g.balanced = 0;
        g.G = 0;
        if (splits > g.nkt) splits = g.nkt;
        g.chunk = (g.nkt + splits - 1) / splits;
        g.eff = (g.nkt + g.chunk - 1) / g.chunk;
        g.slots = g.eff;
    }
}

// Kernel parameters of a decode launch (workspace pointers left null).
attn::DecodeParams decode_params(int B, int H, int H_kv, int Tq, int Tk, int causal, float scale,
                                 const DecGeom &g)
{
    attn::DecodeParams p;
    p.part_o = nullptr;
    p.part_lse = nullptr;
    p.nrows = (long long)B * H * Tq;
    p.H = H;
    p.H_kv = H_kv;
    p.group = H / H_kv;
    p.Tq = Tq;
    p.Tk = Tk;
    p.causal = causal;
    p.rows = p.group * Tq;
    p.nrb = g.nrb;
    p.nkt = g.nkt;
    p.copies = g.copies;
    p.balanced = g.balanced;
    p.chunk = g.chunk;
    p.splits = g.eff;
    p.tot = g.tot;
    p.G = g.G;
    p.c_log2 = scale * 1.4426950408889634f;
    p.limit_ns = kWaitLimitNs;
    return p;
}

template <int D>
int launch_decode(const void *q, const void *k, const void *v, void *o, float *lse, void *ws,
                  int B, int H, int H_kv, int Tq, int Tk, int causal, float scale, int splits,
                  cudaStream_t stream, int sms)
{
    using C = attn::DecCfg<D>;
    DecGeom g;
    decode_geometry(B, H, H_kv, Tq, Tk, splits, sms, g);
    const long long nrows = (long long)B * H * Tq;
    CUtensorMap mq, mk, mv;
    // the Q box is one copy of the rows: 128 / copies rows
    if (make_map(&mq, q, D, (uint64_t)nrows, 1, 128 / g.copies) ||
        make_map(&mk, k, D, Tk, (uint64_t)B * H_kv, 128) ||
        make_map(&mv, v, D, Tk, (uint64_t)B * H_kv, 128))
        return ATTN_ERR_LAUNCH;
    attn::DecodeParams p = decode_params(B, H, H_kv, Tq, Tk, causal, scale, g);
    p.part_o = static_cast<float *>(ws);
    p.part_lse = p.part_o + (size_t)g.slots * g.copies * nrows * D;
    const dim3 grid = g.balanced ? dim3((unsigned)g.G, 1, 1) : dim3(g.eff, B * H_kv, g.nrb);
    if (g.copies == 4)
        attn::decode_partial_kernel<D, 4><<<grid, C::THREADS, C::SMEM, stream>>>(mq, mk, mv, p);
    else if (g.copies == 2)
        attn::decode_partial_kernel<D, 2><<<grid, C::THREADS, C::SMEM, stream>>>(mq, mk, mv, p);
    else
        attn::decode_partial_kernel<D, 1><<<grid, C::THREADS, C::SMEM, stream>>>(mq, mk, mv, p);
    if (launch_status()) return ATTN_ERR_LAUNCH;
    // The merge is launched as a programmatic dependent of the partial kernel:
    // its launch overlaps the partial kernel's tail and it waits on the device
    // (griddepcontrol.wait) until every partial result is written.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((nrows + (128 / D) - 1) / (128 / D)));  // 128 / D rows per CTA
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, attn::decode_combine_kernel<D>, p,
                           static_cast<__nv_bfloat16 *>(o), lse) != cudaSuccess)
        return ATTN_ERR_LAUNCH;
    return launch_status();
}

}  // namespace

extern "C" {

size_t attn_decode_workspace_bytes(int B, int H, int H_kv, int Tq, int Tk, int d_h, int splits)
{
    if (B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || Tq < 1 || Tk < Tq ||
        (d_h != 64 && d_h != 128))
        return 0;
    int sms = 0;
    if (splits <= 0 && device_ready(&sms)) return 0;
    DecGeom g;
    decode_geometry(B, H, H_kv, Tq, Tk, splits, sms, g);
    return (size_t)g.slots * g.copies * B * H * Tq * (size_t)(d_h + 1) * 4;
}

int attn_fwd_decode(const void *q, const void *k, const void *v, void *o, float *lse, void *ws,
                    int B, int H, int H_kv, int Tq, int Tk, int d_h, int causal, float scale,
                    int splits, void *stream)
{
    int rc = validate(q, k, v, o, lse, B, H, Tq, d_h, causal, scale);
    if (rc) return rc;
    if (!ws) return ATTN_ERR_NULL;
    if (misaligned(ws)) return ATTN_ERR_ALIGN;
    if (H_kv < 1 || H % H_kv != 0 || Tk < Tq || (long long)B * H_kv > 65535 ||
        ((long long)(H / H_kv) * Tq + 127) / 128 > 65535 ||
        (long long)B * H * Tq > INT_MAX || (long long)B * H_kv * Tk > INT_MAX)
        return ATTN_ERR_BAD_SHAPE;
    int sms = 0;
    if ((rc = device_ready(&sms))) return rc;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d_h == 64
               ? launch_decode<64>(q, k, v, o, lse, ws, B, H, H_kv, Tq, Tk, causal, scale, splits, s, sms)
               : launch_decode<128>(q, k, v, o, lse, ws, B, H, H_kv, Tq, Tk, causal, scale, splits, s, sms);
}


size_t attn_bwd_workspace_bytes(int B, int H, int T)
{
    if (B < 1 || H < 1 || T < 1 || T > INT_MAX - 128) return 0;
    const size_t Tp = (size_t)((T + 127) / 128) * 128;  // per-row statistics, 128-row blocks
    return (size_t)B * H * Tp * 8;
}

int attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
             const void *dout, void *dq, void *dk, void *dv, void *ws, int B, int H, int H_kv,
             int T, int d_h, int causal, float scale, void *stream)
{
    int rc = validate(q, k, v, o, lse, B, H, T, d_h, causal, scale);
    if (rc) return rc;
    if (!dout || !dq || !dk || !dv || !ws) return ATTN_ERR_NULL;
    if (misaligned(dout) || misaligned(dq) || misaligned(dk) || misaligned(dv) || misaligned(ws))
        return ATTN_ERR_ALIGN;
    if (H_kv < 1 || H % H_kv != 0 || (long long)B * H > 65535 ||
        (long long)B * H * (((long long)T + 127) / 128 * 128) > (long long)INT_MAX)
        return ATTN_ERR_BAD_SHAPE;
    if ((rc = device_ready(nullptr))) return rc;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d_h == 64
               ? launch_bwd<64>(q, k, v, o, lse, dout, dq, dk, dv, ws, B, H, H_kv, T, causal, scale, s)
               : launch_bwd<128>(q, k, v, o, lse, dout, dq, dk, dv, ws, B, H, H_kv, T, causal, scale, s);
}


int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int T,
             int d_h, int causal, float scale, void *stream)
{
    int rc = validate(q, k, v, o, lse, B, H, T, d_h, causal, scale);
    if (rc) return rc;
    int sms = 0;
    if ((rc = device_ready(&sms))) return rc;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d_h == 64 ? launch_fused<64>(q, k, v, o, lse, B, H, H, T, causal, scale, s, sms)
                     : launch_fused<128>(q, k, v, o, lse, B, H, H, T, causal, scale, s, sms);
}

int attn_fwd_gqa(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
                 int H_kv, int T, int d_h, int causal, float scale, void *stream)
{
    int rc = validate(q, k, v, o, lse, B, H, T, d_h, causal, scale);
    if (rc) return rc;
    if (H_kv < 1 || H % H_kv != 0) return ATTN_ERR_BAD_SHAPE;
    int sms = 0;
    if ((rc = device_ready(&sms))) return rc;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d_h == 64 ? launch_fused<64>(q, k, v, o, lse, B, H, H_kv, T, causal, scale, s, sms)
                     : launch_fused<128>(q, k, v, o, lse, B, H, H_kv, T, causal, scale, s, sms);
}

size_t attn_unfused_workspace_bytes(int B, int H, int T)
{
    if (B < 1 || H < 1 || T < 1) return 0;
    const unsigned long long n = (unsigned long long)B * H * T * (unsigned long long)T * 2ull;
    return (size_t)n;
}

int attn_fwd_unfused(const void *q, const void *k, const void *v, void *o, float *lse, void *s_ws,
                     void *p_ws, int B, int H, int T, int d_h, int causal, float scale,
                     void *stream)
{
    int rc = validate(q, k, v, o, lse, B, H, T, d_h, causal, scale);
    if (rc) return rc;
    if (!s_ws || !p_ws) return ATTN_ERR_NULL;
    if (misaligned(s_ws) || misaligned(p_ws)) return ATTN_ERR_ALIGN;
    if (T % 128 != 0 || (long long)B * H > 65535) return ATTN_ERR_BAD_SHAPE;
    int sms = 0;
    if ((rc = device_ready(&sms))) return rc;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d_h == 64 ? launch_unfused<64>(q, k, v, o, lse, s_ws, p_ws, B * H, T, causal, scale, s, sms)
                     : launch_unfused<128>(q, k, v, o, lse, s_ws, p_ws, B * H, T, causal, scale, s, sms);
}

int attn_fwd_host(const void *q_host, const void *k_host, const void *v_host, void *o_host,
                  float *lse_host, void *dq, void *dk, void *dv, void *do_, float *dlse, int B,
                  int H, int T, int d_h, int causal, float scale, void *stream)
{
    if (!q_host || !k_host || !v_host || !o_host || !lse_host) return ATTN_ERR_NULL;
    int rc = validate(dq, dk, dv, do_, dlse, B, H, T, d_h, causal, scale);
    if (rc) return rc;
    if ((rc = device_ready(nullptr))) return rc;
    HostPipe *hp = host_pipe();
    if (!hp) return ATTN_ERR_LAUNCH;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Heads are independent: cut the B * H heads into chunks and overlap the
    // host -> device copy of chunk c + 1, the attention of chunk c (on
    // `stream`) and the device -> host copy of chunk c - 1 (the two copy
    // directions run on separate copy engines).
    const int bh = B * H;
    const int nch = bh < kHostChunks ? bh : kHostChunks;
    const int per = (bh + nch - 1) / nch;
    const size_t head = (size_t)T * d_h;  // elements of one head
    auto cp = [](void *dst, const void *src, size_t bytes, cudaMemcpyKind kind, cudaStream_t st) {
        return cudaMemcpyAsync(dst, src, bytes, kind, st) == cudaSuccess;
    };
    bool ok = cudaEventRecord(hp->start, s) == cudaSuccess &&  // earlier work on the buffers
              cudaStreamWaitEvent(hp->in, hp->start, 0) == cudaSuccess &&
              cudaStreamWaitEvent(hp->out, hp->start, 0) == cudaSuccess;
    for (int c = 0; ok && c < nch; ++c) {
        const int h0 = c * per, nh = (h0 + per <= bh ? per : bh - h0);
        if (nh <= 0) break;
        const size_t off = (size_t)h0 * head * 2, bytes = (size_t)nh * head * 2;
        ok = cp(static_cast<char *>(dq) + off, static_cast<const char *>(q_host) + off, bytes,
                cudaMemcpyHostToDevice, hp->in) &&
             cp(static_cast<char *>(dk) + off, static_cast<const char *>(k_host) + off, bytes,
                cudaMemcpyHostToDevice, hp->in) &&
             cp(static_cast<char *>(dv) + off, static_cast<const char *>(v_host) + off, bytes,
                cudaMemcpyHostToDevice, hp->in) &&
             cudaEventRecord(hp->loaded[c], hp->in) == cudaSuccess;
    }
    int fail = ATTN_OK;
    for (int c = 0; ok && c < nch; ++c) {
        const int h0 = c * per, nh = (h0 + per <= bh ? per : bh - h0);
        if (nh <= 0) break;
        const size_t off = (size_t)h0 * head * 2, bytes = (size_t)nh * head * 2;
        const size_t loff = (size_t)h0 * T * sizeof(float), lbytes = (size_t)nh * T * sizeof(float);
        if (!(ok = cudaStreamWaitEvent(s, hp->loaded[c], 0) == cudaSuccess)) break;
        if ((fail = attn_fwd(static_cast<const char *>(dq) + off, static_cast<const char *>(dk) + off,
                             static_cast<const char *>(dv) + off, static_cast<char *>(do_) + off,
                             reinterpret_cast<float *>(reinterpret_cast<char *>(dlse) + loff), 1, nh,
                             T, d_h, causal, scale, stream)))
            break;
        ok = cudaEventRecord(hp->computed[c], s) == cudaSuccess &&
             cudaStreamWaitEvent(hp->out, hp->computed[c], 0) == cudaSuccess &&
             cp(static_cast<char *>(o_host) + off, static_cast<const char *>(do_) + off, bytes,
                cudaMemcpyDeviceToHost, hp->out) &&
             cp(reinterpret_cast<char *>(lse_host) + loff, reinterpret_cast<const char *>(dlse) + loff,
                lbytes, cudaMemcpyDeviceToHost, hp->out);
    }
    // `stream` completes only after every copy queued above, on success and on
    // failure alike, so the caller's buffers are not in use once it has
    // drained (a wait uses the event's most recent record at the time of the
    // call, so one event serves both streams in turn)
    const bool joined = cudaEventRecord(hp->done, hp->in) == cudaSuccess &&
                        cudaStreamWaitEvent(s, hp->done, 0) == cudaSuccess &&
                        cudaEventRecord(hp->done, hp->out) == cudaSuccess &&
                        cudaStreamWaitEvent(s, hp->done, 0) == cudaSuccess;
    if (fail != ATTN_OK) return fail;
    if (!ok || !joined) {
        (void)cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    return ATTN_OK;
}

int attn_last_error(void)
{
    if (cudaDeviceSynchronize() != cudaSuccess) {
        (void)cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    unsigned int v = 0, w = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, attn::g_status, sizeof v) != cudaSuccess ||
        cudaMemcpyFromSymbol(&w, attn::g_status_where, sizeof w) != cudaSuccess ||
        cudaMemcpyToSymbol(attn::g_status, &zero, sizeof zero) != cudaSuccess ||
        cudaMemcpyToSymbol(attn::g_status_where, &zero, sizeof zero) != cudaSuccess) {
        (void)cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    g_last_where = w;
    return (int)v;
}

const char *attn_status_str(int status)
{
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_NULL: return "null pointer";
        case ATTN_ERR_UNSUPPORTED_DH: return "unsupported head dimension (64 or 128)";
        case ATTN_ERR_BAD_SHAPE: return "bad shape";
        case ATTN_ERR_ALIGN: return "pointer under-aligned (tensors 16 bytes, lse 4 bytes)";
        case ATTN_ERR_BAD_SCALE: return "scale not finite and positive";
        case ATTN_ERR_LAUNCH: return "CUDA launch or runtime error";
        case ATTN_ERR_TIMEOUT: return "device wait timed out";
        case ATTN_ERR_NO_DEVICE: return "no sm_100 device";
        case ATTN_ERR_BAD_ARG: return "bad argument";
        case ATTN_ERR_WORKSPACE_LIMIT: return "problem exceeds the static workspace (B*H*T*T > 16777216)";
        default: return "unknown status";
    }
}

int attn_fused_grid_ctas(int B, int H, int T, int d_h, int causal)
{
    if (B < 1 || H < 1 || T < 1 || (d_h != 64 && d_h != 128)) return 0;
    int sms = 0;
    if (device_ready(&sms)) return 0;
    return fused_grid((long long)B * H, T, causal ? 1 : 0, sms);
}

const char *attn_version(void) { return "0.1.0"; }

// ------------------------------------------------------------------ self-tests
int attn_selftest_qk_tile(const void *q, const void *k, float *s, int d_h, void *stream)
{
    if (!q || !k || !s) return ATTN_ERR_NULL;
    if (d_h != 64 && d_h != 128) return ATTN_ERR_UNSUPPORTED_DH;
    if (misaligned(q) || misaligned(k) || misaligned(s)) return ATTN_ERR_ALIGN;
    int rc = device_ready(nullptr);
    if (rc) return rc;
    CUtensorMap mq, mk;
    if (make_map(&mq, q, d_h, 128, 1, 128) || make_map(&mk, k, d_h, 128, 1, 128))
        return ATTN_ERR_LAUNCH;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d_h == 64)
        attn::selftest_qk_kernel<64><<<1, 128, 1024 + 2 * 128 * 64 * 2 + 64, st>>>(mq, mk, s,
                                                                                 kWaitLimitNs);
    else
        attn::selftest_qk_kernel<128><<<1, 128, 1024 + 2 * 128 * 128 * 2 + 64, st>>>(mq, mk, s,
                                                                                   kWaitLimitNs);
    return launch_status();
}

int attn_selftest_pv_tile(const void *p, const void *v, float *o, int d_h, void *stream)
{
    if (!p || !v || !o) return ATTN_ERR_NULL;
    if (d_h != 64 && d_h != 128) return ATTN_ERR_UNSUPPORTED_DH;
    if (misaligned(p) || misaligned(v) || misaligned(o)) return ATTN_ERR_ALIGN;
    int rc = device_ready(nullptr);
    if (rc) return rc;
    CUtensorMap mv;
    if (make_map(&mv, v, d_h, 128, 1, 128)) return ATTN_ERR_LAUNCH;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const auto *pp = static_cast<const __nv_bfloat16 *>(p);
    if (d_h == 64)
        attn::selftest_pv_kernel<64><<<1, 128, 1024 + 128 * 64 * 2 + 64, st>>>(pp, mv, o,
                                                                             kWaitLimitNs);
    else
        attn::selftest_pv_kernel<128><<<1, 128, 1024 + 128 * 128 * 2 + 64, st>>>(pp, mv, o,
                                                                               kWaitLimitNs);
    return launch_status();
}

int attn_selftest_timeout(int limit_us, void *stream)
{
    if (limit_us < 1 || limit_us > 1000000) return ATTN_ERR_BAD_ARG;
    int rc = device_ready(nullptr);
    if (rc) return rc;
    attn::selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)limit_us * 1000ull);
    return launch_status();
}

int attn_selftest_set_mma_order(int mode)
{
    if (mode != 0 && mode != 1) return -1;
    const int prev = g_mma_order;
    g_mma_order = mode;
    return prev;
}

int attn_selftest_last_wait_site(void) { return (int)g_last_where; }

int attn_selftest_fused_plan(int B, int H, int H_kv, int T, int causal, int sms, int *units,
                             int cap, int *ctas)
{
    if (B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || T < 1 || sms < 1 ||
        (causal != 0 && causal != 1) || (long long)B * H * (long long)T > (long long)INT_MAX)
        return -1;
    const attn::FusedParams p = fused_params(B, H, H_kv, T, causal, 1.f);
    const int G = fused_grid((long long)B * H, T, causal, sms);
    if (ctas) *ctas = G;
    long long nrec = 0;
    for (int c = 0; c < G; ++c) {
        attn::UnitInfo u;
        for (int k = 0;; ++k) {
            const int r = attn::unit_of_cta(p, G, c, k, u);
            if (r < 0) break;
            if (r == 0) continue;
            if (units && nrec < cap) {
                int *x = units + 7 * nrec;
                x[0] = c; x[1] = k; x[2] = u.bh; x[3] = u.kvh; x[4] = u.i0; x[5] = u.n[0]; x[6] = u.n[1];
            }
            ++nrec;
        }
    }
    return nrec > INT_MAX ? INT_MAX : (int)nrec;
}

int attn_selftest_decode_plan(int B, int H, int H_kv, int Tq, int Tk, int splits, int sms,
                              int *segs, int seg_cap, int *nseg, int nseg_cap, int *slots,
                              int *copies)
{
    if (B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || Tq < 1 || Tk < Tq || sms < 1 ||
        (long long)B * H_kv > 65535 || (long long)B * H * Tq > INT_MAX)
        return -1;
    DecGeom g;
    decode_geometry(B, H, H_kv, Tq, Tk, splits, sms, g);
    const attn::DecodeParams p = decode_params(B, H, H_kv, Tq, Tk, 1, 1.f, g);
    const int gx = g.balanced ? g.G : g.eff, gy = g.balanced ? 1 : B * H_kv, gz = g.balanced ? 1 : g.nrb;
    long long nrec = 0;
    for (int bz = 0; bz < gz; ++bz)
        for (int by = 0; by < gy; ++by)
            for (int bx = 0; bx < gx; ++bx) {
                attn::DecSeg sg;
                for (int idx = 0; attn::dec_segment(p, bx, by, bz, idx, sg); ++idx, ++nrec) {
                    if (!segs || nrec >= seg_cap) continue;
                    int *r = segs + 8 * nrec;
                    r[0] = bx; r[1] = by; r[2] = bz;
                    r[3] = sg.kvbh; r[4] = sg.qt; r[5] = sg.t0; r[6] = sg.n; r[7] = sg.slot * g.copies;
                }
            }
    const long long W = (long long)B * H_kv * g.nrb;
    for (long long w = 0; nseg && w < W && w < nseg_cap; ++w)
        nseg[w] = (g.balanced ? attn::dec_nseg(w, g.nkt, g.tot, g.G) : g.eff) * g.copies;
    if (slots) *slots = g.slots * g.copies;
    if (copies) *copies = g.copies;
    return nrec > INT_MAX ? INT_MAX : (int)nrec;
}

int attn_selftest_set_exp_split(int pairs_of_8)
{
    if (pairs_of_8 != -1 && pairs_of_8 != 0 && pairs_of_8 != 2 && pairs_of_8 != 3 &&
        pairs_of_8 != 4)
        return -2;
    const int prev = g_exp_split;
    g_exp_split = pairs_of_8;
    return prev;
}

}  // extern "C"

// ------------------------------------------------------------ allocation-free unfused forward
// Callers that cannot allocate device memory (a plug-in whose host owns the
// device through its own memory pool, or code that must not risk the
// synchronisation an allocation or free can cause) get S and P from this
// static array instead of caller-provided workspaces: 64 MiB, S in the first
// half and P in the second.  Every GPU that loads the library reserves it
// until the process exits.  In host code the symbol is only a host-side
// stand-in; its device address is looked up per device (below) and passed to
// the kernels.
constexpr size_t kNoallocBytes = (size_t)64 << 20;
static __device__ __align__(256) unsigned char g_noalloc_ws[kNoallocBytes];

extern "C" int attn_fwd_unfused_noalloc(const void *q, const void *k, const void *v, void *o,
                                        float *lse, int B, int H, int T, int d_h, int causal,
                                        float scale, void *stream)
{
    int rc = validate(q, k, v, o, lse, B, H, T, d_h, causal, scale);
    if (rc) return rc;
    if (T % 128 != 0 || (long long)B * H > 65535) return ATTN_ERR_BAD_SHAPE;
    const unsigned long long one = (unsigned long long)B * H * T * (unsigned long long)T * 2ull;
    if (one > kNoallocBytes / 2) return ATTN_ERR_WORKSPACE_LIMIT;
    int sms = 0;
    if ((rc = device_ready(&sms))) return rc;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        (void)cudaGetLastError();
        return ATTN_ERR_NO_DEVICE;
    }
    DeviceState &st = g_dev[dev];
    if (st.noalloc_ws == nullptr) {  // first call on this device (in this context)
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_ws) != cudaSuccess || ptr == nullptr) {
            (void)cudaGetLastError();
            return ATTN_ERR_LAUNCH;
        }
        st.noalloc_ws = ptr;
    }
    auto *ws = static_cast<unsigned char *>(st.noalloc_ws);
    void *s_ws = ws;
    void *p_ws = ws + kNoallocBytes / 2;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d_h == 64 ? launch_unfused<64>(q, k, v, o, lse, s_ws, p_ws, B * H, T, causal, scale, s, sms)
                     : launch_unfused<128>(q, k, v, o, lse, s_ws, p_ws, B * H, T, causal, scale, s, sms);
}
