// yarnattn.cu -- the C ABI of libyarnattn.so: argument checks, TMA descriptor
// set-up and kernel launches on the caller's stream.  All kernels live in this
// translation unit (they share the device status word).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>

#include "../../include/yarnattn.h"
#include "decode_sm100.cuh"
#include "kvprep_sm100.cuh"
#include "merge_sm100.cuh"
#include "prefill_sm100.cuh"

namespace yr_host {

thread_local std::string g_err;
void set_error(const std::string &msg) { g_err = msg; }

int fail(int code, const std::string &msg) {
    set_error(msg);
    return code;
}

int cuda_fail(const char *what, cudaError_t e) {
    return fail(YR_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

uint64_t wait_timeout_ns() {
    static uint64_t ns = [] {
        const char *s = std::getenv("YR_WAIT_TIMEOUT_MS");
        long ms = s ? std::strtol(s, nullptr, 10) : 2000;
        if (ms < 1) ms = 1;
        return static_cast<uint64_t>(ms) * 1000000ull;
    }();
    return ns;
}

// The context current on the calling thread.  The CUDA runtime launches into it, and
// function attributes and the addresses of module globals belong to it, so the
// one-time set-up below is kept per context (a host application may make a context
// of its own current, or reset the device, between calls).
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

template <typename Fn>
Fn driver_entry(const char *name) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<Fn>(ptr);
    return nullptr;
}

int current_context(int *dev_out, unsigned long long *ctx_id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        get_current = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
        get_id = driver_entry<CtxGetIdFn>("cuCtxGetId");
    });
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (!get_current || !get_id)
        return fail(YR_ECUDA, "cuCtxGetCurrent/cuCtxGetId are not available from the driver");
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS)
        return fail(YR_ECUDA, "cuCtxGetCurrent failed");
    if (ctx == nullptr) {
        // No context yet on this thread: the runtime would make the device's primary
        // context current at its next call; make it current now so it can be named.
        e = cudaSetDevice(dev);
        if (e != cudaSuccess) return cuda_fail("cudaSetDevice", e);
        if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
            return fail(YR_ECUDA, "no CUDA context is current");
    }
    if (get_id(ctx, ctx_id) != CUDA_SUCCESS) return fail(YR_ECUDA, "cuCtxGetId failed");
    *dev_out = dev;
    return YR_OK;
}

// Per-context one-time set-up: architecture check and shared-memory opt-in.
struct DeviceState {
    bool sm100 = false;
    bool prefill_regs_ok = false;  // launched register count covers the setmaxnreg split
    int sm_count = 0;
};
std::mutex g_dev_mu;
std::unordered_map<unsigned long long, DeviceState> g_dev;  // by context id

int prepare_device(int *sm_count, DeviceState *out = nullptr) {
    int dev = 0;
    unsigned long long ctx = 0;
    int rc = current_context(&dev, &ctx);
    if (rc != YR_OK) return rc;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    auto it = g_dev.find(ctx);
    if (it == g_dev.end()) {
        DeviceState st;
        cudaDeviceProp prop;
        cudaError_t e = cudaGetDeviceProperties(&prop, dev);
        if (e != cudaSuccess) return cuda_fail("cudaGetDeviceProperties", e);
        st.sm100 = (prop.major == 10 && prop.minor == 0);
        st.sm_count = prop.multiProcessorCount;
        if (st.sm100) {
            struct {
                const void *fn;
                size_t bytes;
            } attrs[] = {
                {reinterpret_cast<const void *>(&yr::prefill_attn_kernel<128, false>),
                 yr::prefill_smem_bytes<128>()},
                {reinterpret_cast<const void *>(&yr::prefill_attn_kernel<128, true>),
                 yr::prefill_smem_bytes<128>()},
                {reinterpret_cast<const void *>(&yr::prefill_attn_kernel<64, false>),
                 yr::prefill_smem_bytes<64>()},
                {reinterpret_cast<const void *>(&yr::prefill_attn_kernel<64, true>),
                 yr::prefill_smem_bytes<64>()},
                {reinterpret_cast<const void *>(&yr::decode_split_kernel<128, 1>),
                 yr::decode_smem_bytes<128>()},
                {reinterpret_cast<const void *>(&yr::decode_split_kernel<128, 2>),
                 yr::decode_smem_bytes<128>()},
                {reinterpret_cast<const void *>(&yr::decode_split_kernel<64, 1>),
                 yr::decode_smem_bytes<64>()},
                {reinterpret_cast<const void *>(&yr::decode_split_kernel<64, 2>),
                 yr::decode_smem_bytes<64>()},
            };
            for (auto &a : attrs) {
                e = cudaFuncSetAttribute(a.fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(a.bytes));
                if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute", e);
            }
            // The prefill kernel re-splits its registers between warpgroups
            // (setmaxnreg); that only works if the launch reserves enough of them.
            st.prefill_regs_ok = true;
            for (const void *fn : {reinterpret_cast<const void *>(&yr::prefill_attn_kernel<128, false>),
                                   reinterpret_cast<const void *>(&yr::prefill_attn_kernel<128, true>),
                                   reinterpret_cast<const void *>(&yr::prefill_attn_kernel<64, false>),
                                   reinterpret_cast<const void *>(&yr::prefill_attn_kernel<64, true>)}) {
                cudaFuncAttributes fa;
                e = cudaFuncGetAttributes(&fa, fn);
                if (e != cudaSuccess) return cuda_fail("cudaFuncGetAttributes", e);
                if (fa.numRegs < yr::kMinLaunchRegs) st.prefill_regs_ok = false;
            }
        }
        it = g_dev.emplace(ctx, st).first;
    }
    const DeviceState &st = it->second;
    if (!st.sm100) return fail(YR_EUNSUPPORTED, "the current device is not sm_100 (B200)");
    if (sm_count) *sm_count = st.sm_count;
    if (out) *out = st;
    return YR_OK;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Element strides {b, h, t}: either given, or contiguous for [B][H][T][d].
void strides_or_contiguous(const int64_t *s, int H, int T, int d, long long out[3]) {
    if (s) {
        out[0] = s[0];
        out[1] = s[1];
        out[2] = s[2];
    } else {
        out[2] = d;
        out[1] = static_cast<long long>(T) * d;
        out[0] = static_cast<long long>(H) * T * d;
    }
}

bool strides_ok(const long long s[3]) {
    for (int i = 0; i < 3; ++i)
        if (s[i] <= 0 || (s[i] % 8) != 0 || s[i] >= (1ll << 38)) return false;
    return true;
}

int encode(CUtensorMap *map, CUtensorMapDataType dt, int rank, const void *base,
           const cuuint64_t *dims, const cuuint64_t *strides_bytes, const cuuint32_t *box,
           const char *what) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(YR_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(map, dt, static_cast<cuuint32_t>(rank), const_cast<void *>(base), dims,
                    strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(YR_ECUDA, std::string("cuTensorMapEncodeTiled failed for ") + what +
                                  " (code " + std::to_string(static_cast<int>(r)) + ")");
    return YR_OK;
}

// Prefill workspace: the rotated keys and the values in fp16.
size_t prefill_ws_bytes(long long B, long long Hkv, long long T, long long d) {
    return static_cast<size_t>(2 * B * Hkv * T * d * 2);
}

// Partial-result slots per (b, KV head): a block of the balanced split holds at least
// kDecChunk keys, so a segment of at most T_max keys touches at most this many blocks.
int decode_parts(int T_max) { return (T_max + yr::kDecChunk - 1) / yr::kDecChunk + 1; }

size_t decode_ws_bytes(long long B, long long Hq, long long Hkv, long long d, int T_max) {
    const long long g = Hq / Hkv;
    return static_cast<size_t>(B * Hkv * decode_parts(T_max) * g * (d + 2) * 4);
}

// Blocks of the split launch: one full wave (resident blocks per SM x SMs), so that the
// equal shares of the balanced split all run at once.
template <int HD, int NT>
int decode_grid(int sm_count) {
    static int per_sm = 0;  // same value on every device of this build's target
    if (per_sm == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, yr::decode_split_kernel<HD, NT>,
                                                          yr::kDecThreads,
                                                          yr::decode_smem_bytes<HD>()) != cudaSuccess ||
            n < 1)
            n = 1;
        per_sm = n;
    }
    return per_sm * sm_count;
}

}  // namespace yr_host

using namespace yr_host;

extern "C" const char *yr_last_error(void) { return g_err.c_str(); }

extern "C" int yr_version(void) { return 1 * 10000 + 0 * 100 + 0; }

extern "C" size_t yr_attn_prefill_workspace_bytes(int B, int Hkv, int T, int d) {
    if (B < 1 || Hkv < 1 || T < 1 || d < 2) return 0;
    return prefill_ws_bytes(B, Hkv, T, d);
}

extern "C" size_t yr_attn_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int T_max) {
    if (B < 1 || Hq < 1 || Hkv < 1 || d < 2 || T_max < 1 || Hq % Hkv) return 0;
    return decode_ws_bytes(B, Hq, Hkv, d, T_max);
}

namespace yr_host {

int check_common(const char *fn, int B, int Hkv, int T, int d, const yr_rope_table *tab,
                 const void *workspace, size_t workspace_bytes) {
    const std::string f(fn);
    if (!tab || !workspace) return fail(YR_EINVAL, f + ": tab and workspace must be non-NULL");
    if (B < 1 || Hkv < 1 || T < 1) return fail(YR_EINVAL, f + ": B, Hkv and T must be >= 1");
    if (d != 64 && d != 128) return fail(YR_EUNSUPPORTED, f + ": d must be 64 or 128");
    if (tab->head_dim != d) return fail(YR_EINVAL, f + ": table head_dim != d");
    if (tab->pairs != YR_PAIR_INTERLEAVED && tab->pairs != YR_PAIR_HALF)
        return fail(YR_EINVAL, f + ": table pairs must be YR_PAIR_INTERLEAVED or YR_PAIR_HALF");
    const size_t need = prefill_ws_bytes(B, Hkv, T, d);
    if (workspace_bytes < need)
        return fail(YR_EINVAL, f + ": workspace too small (need " + std::to_string(need) + " bytes)");
    if (!aligned(workspace, 256)) return fail(YR_EINVAL, f + ": workspace must be 256-byte aligned");
    return YR_OK;
}

int check_prepare(const void *k, const void *v, const void *k_cache, const float *k_rot_dbg,
                  int B, int Hkv, int T, int d, const int64_t *k_strides, const int64_t *v_strides,
                  const int64_t *kc_strides, const yr_rope_table *tab, const void *workspace,
                  size_t workspace_bytes, const char *fn, long long ks[3], long long vs[3],
                  long long cs[3]) {
    if (!k || !v) return fail(YR_EINVAL, std::string(fn) + ": k and v must be non-NULL");
    int rc = check_common(fn, B, Hkv, T, d, tab, workspace, workspace_bytes);
    if (rc != YR_OK) return rc;
    for (const void *ptr : {k, v, k_cache, static_cast<const void *>(k_rot_dbg)})
        if (ptr && !aligned(ptr, 16))
            return fail(YR_EINVAL, std::string(fn) + ": pointers must be 16-byte aligned");
    strides_or_contiguous(k_strides, Hkv, T, d, ks);
    strides_or_contiguous(v_strides, Hkv, T, d, vs);
    strides_or_contiguous(kc_strides, Hkv, T, d, cs);
    if (!strides_ok(ks) || !strides_ok(vs) || (k_cache && !strides_ok(cs)))
        return fail(YR_EINVAL, std::string(fn) + ": strides must be positive multiples of 8 elements");
    return YR_OK;
}

int check_attend(const void *q, const void *o, const float *lse, const float *q_rot_dbg, int B,
                 int Hq, int Hkv, int T, int d, const int64_t *q_strides, const int64_t *o_strides,
                 const yr_rope_table *tab, int causal, int window, int n_sink,
                 const void *workspace, size_t workspace_bytes, const char *fn, long long qs[3],
                 long long os[3]) {
    const std::string f(fn);
    if (!q || !o) return fail(YR_EINVAL, f + ": q and o must be non-NULL");
    if (Hq < 1) return fail(YR_EINVAL, f + ": B, Hq, Hkv and T must be >= 1");
    int rc = check_common(fn, B, Hkv, T, d, tab, workspace, workspace_bytes);
    if (rc != YR_OK) return rc;
    if (Hq % Hkv != 0) return fail(YR_EINVAL, f + ": Hq must be a multiple of Hkv");
    if (causal != 0 && causal != 1) return fail(YR_EINVAL, f + ": causal must be 0 or 1");
    if (window < 0 || n_sink < 0) return fail(YR_EINVAL, f + ": window and n_sink must be >= 0");
    if (window > 0 && !causal) return fail(YR_EINVAL, f + ": a window needs causal=1");
    if (n_sink > 0 && window == 0) return fail(YR_EINVAL, f + ": sinks need a window");
    if (static_cast<long long>(B) * Hq * ((T + 255) / 256) * 16 >= (1ll << 31))
        return fail(YR_EINVAL, f + ": problem too large for one launch");
    for (const void *ptr : {q, o, static_cast<const void *>(q_rot_dbg)})
        if (ptr && !aligned(ptr, 16)) return fail(YR_EINVAL, f + ": pointers must be 16-byte aligned");
    if (lse && !aligned(lse, 4)) return fail(YR_EINVAL, f + ": lse must be 4-byte aligned");
    strides_or_contiguous(q_strides, Hq, T, d, qs);
    strides_or_contiguous(o_strides, Hq, T, d, os);
    if (!strides_ok(qs) || !strides_ok(os))
        return fail(YR_EINVAL, f + ": strides must be positive multiples of 8 elements");
    return YR_OK;
}

int launch_prepare(const void *k, const void *v, void *k_cache, float *k_rot_dbg, int B, int Hkv,
                   int T, int d, const long long ks[3], const long long vs[3],
                   const long long cs[3], const yr_rope_table *tab, void *workspace,
                   int sm_count, cudaStream_t st, int pos0 = 0) {
    __half *k16 = static_cast<__half *>(workspace);
    __half *v16 = k16 + static_cast<size_t>(B) * Hkv * T * d;
    yr::KvPrepParams kp;
    std::memset(&kp, 0, sizeof kp);
    kp.k = static_cast<const __nv_bfloat16 *>(k);
    kp.v = static_cast<const __nv_bfloat16 *>(v);
    kp.ksb = ks[0]; kp.ksh = ks[1]; kp.kst = ks[2];
    kp.vsb = vs[0]; kp.vsh = vs[1]; kp.vst = vs[2];
    kp.k16 = k16;
    kp.v16 = v16;
    kp.kc = static_cast<__nv_bfloat16 *>(k_cache);
    kp.csb = cs[0]; kp.csh = cs[1]; kp.cst = cs[2];
    kp.k_dbg = k_rot_dbg;
    kp.Hkv = Hkv; kp.T = T; kp.d = d;
    kp.pos0 = pos0;
    const bool half = tab->pairs == YR_PAIR_HALF;
    kp.n_items = static_cast<long long>(B) * Hkv * T * (half ? d / 16 : d / 8);
    for (int i = 0; i < d / 2; ++i) kp.turns[i] = tab->turns[i];
    long long blocks = (kp.n_items + 255) / 256;
    const long long cap = static_cast<long long>(sm_count) * 16;
    if (blocks > cap) blocks = cap;
    if (half)
        yr::kv_prep_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(kp);
    else
        yr::kv_prep_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(kp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("kv_prep_kernel launch", e);
    return YR_OK;
}

// The fp16 rotated keys and values the attention kernel reads: planes of ld16 rows
// of d elements, one per (b, KV head), keys [0, Tk) of each.
struct KvPlanes {
    const __half *k16;
    const __half *v16;
    long long ld16;
};
// The layout of a prefill workspace: K [B*Hkv][Tk][d], then V the same.
KvPlanes workspace_planes(const void *workspace, int B, int Hkv, int Tk, int d) {
    const __half *k16 = static_cast<const __half *>(workspace);
    return {k16, k16 + static_cast<size_t>(B) * Hkv * Tk * d, Tk};
}

// Does the attention kernel pair two query heads per CTA, and how many (batch, head unit,
// query block) items does a call of T rows have?  Pairs need an even number of query heads
// per KV head.  They pay off with a window, where a CTA's key tiles are few and the two
// tiles a 256-row block has for one of its halves alone (the window's first, the
// diagonal's last) are a large share of them: +1-4% on the windowed 64K GQA workloads,
// -0.4% / -1% on the dense 128K / 64K ones (four alternating rounds on one B200).
int attend_head_pair(int Hq, int Hkv, int window) {
    return window > 0 && (Hq / Hkv) % 2 == 0 ? 1 : 0;
}
long long attend_items(int B, int Hq, int Hkv, int T, int window) {
    return attend_head_pair(Hq, Hkv, window)
               ? static_cast<long long>(B) * (Hq / 2) * ((T + 127) / 128)
               : static_cast<long long>(B) * Hq * ((T + 255) / 256);
}

// T query rows against the Tk keys of `kv`.  Key n sits at position k_pos0 + n and
// query row r at k_pos0 + q_off + r; masks use the offsets relative to key 0.
int launch_attend(const void *q, void *o, float *lse, float *q_rot_dbg, int B, int Hq, int Hkv,
                  int T, int d, const long long qs[3], const long long os[3],
                  const yr_rope_table *tab, int causal, int window, int n_sink,
                  const KvPlanes &kv, cudaStream_t st, int Tk, int q_off, int k_pos0 = 0,
                  float *o32 = nullptr, int n_split = 1) {
    DeviceState ds;
    int rc = prepare_device(nullptr, &ds);
    if (rc != YR_OK) return rc;
    if (!ds.prefill_regs_ok)
        return fail(YR_EUNSUPPORTED, "prefill kernel was built with too few registers per thread "
                                     "for its warpgroup register split");
    yr::PrefillParams pp;
    std::memset(&pp, 0, sizeof pp);
    {
        const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T),
                                    static_cast<cuuint64_t>(Hq), static_cast<cuuint64_t>(B)};
        const cuuint64_t strides[3] = {static_cast<cuuint64_t>(qs[2] * 2),
                                       static_cast<cuuint64_t>(qs[1] * 2),
                                       static_cast<cuuint64_t>(qs[0] * 2)};
        const cuuint32_t box[4] = {64, 128, 1, 1};
        rc = encode(&pp.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, q, dims, strides, box, "q");
        if (rc != YR_OK) return rc;
    }
    {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(Tk),
                                    static_cast<cuuint64_t>(B) * Hkv};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                       static_cast<cuuint64_t>(kv.ld16) * d * 2};
        const cuuint32_t box[3] = {64, 128, 1};
        rc = encode(&pp.tm_k, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, kv.k16, dims, strides, box,
                    "rotated k");
        if (rc != YR_OK) return rc;
        rc = encode(&pp.tm_v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, kv.v16, dims, strides, box, "v");
        if (rc != YR_OK) return rc;
    }
    pp.o = static_cast<__nv_bfloat16 *>(o);
    pp.osb = os[0]; pp.osh = os[1]; pp.ost = os[2];
    pp.o32 = o32;
    pp.lse = lse;
    pp.q_dbg = q_rot_dbg;
    pp.B = B; pp.Hq = Hq; pp.Hkv = Hkv; pp.T = T; pp.group = Hq / Hkv;
    pp.Tk = Tk; pp.q_off = q_off; pp.k_pos0 = k_pos0;
    pp.causal = causal; pp.window = window; pp.n_sink = n_sink;
    // Windowed calls with an even number of query heads per KV head: a CTA takes two heads of
    // one group at the same 128 rows, so both query tiles see the same key tiles.
    pp.head_pair = attend_head_pair(Hq, Hkv, window);
    pp.n_qblocks = pp.head_pair ? (T + 127) / 128 : (T + 255) / 256;
    pp.n_split = n_split;
    pp.split_rows = static_cast<long long>(B) * Hq * T;
    // Grouped query heads read each K/V tile several times: order the CTAs by KV head
    // so that re-reads hit L2 (measured: +2.7% at the 128K GQA workload, neutral for MHA).
    pp.kv_major = pp.group > 1 ? 1 : 0;
    pp.alibi = tab->method == YR_ALIBI ? 1 : 0;
    const bool half = tab->pairs == YR_PAIR_HALF;
    pp.sl2 = static_cast<float>(tab->softmax_scale * 1.4426950408889634);
    pp.timeout_ns = wait_timeout_ns();
#ifdef YR_FAULT_HOOKS
    // Test build only: the failure-path hook, read on every launch.
    const char *drop = std::getenv("YR_FAULT_DROP_KV_TILE");
    pp.fault_drop_tile = drop ? static_cast<int>(std::strtol(drop, nullptr, 10)) : -1;
#else
    pp.fault_drop_tile = -1;
#endif
    for (int i = 0; i < d / 2; ++i) pp.turns[i] = tab->turns[i];
    const unsigned grid =
        static_cast<unsigned>(attend_items(B, Hq, Hkv, T, window) * n_split);
    if (d == 128 && !half)
        yr::prefill_attn_kernel<128, false>
            <<<grid, yr::kPrefillThreads, yr::prefill_smem_bytes<128>(), st>>>(pp);
    else if (d == 128)
        yr::prefill_attn_kernel<128, true>
            <<<grid, yr::kPrefillThreads, yr::prefill_smem_bytes<128>(), st>>>(pp);
    else if (!half)
        yr::prefill_attn_kernel<64, false>
            <<<grid, yr::kPrefillThreads, yr::prefill_smem_bytes<64>(), st>>>(pp);
    else
        yr::prefill_attn_kernel<64, true>
            <<<grid, yr::kPrefillThreads, yr::prefill_smem_bytes<64>(), st>>>(pp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("prefill_attn_kernel launch", e);
    return YR_OK;
}

}  // namespace yr_host

extern "C" int yr_prefill_prepare_kv(const void *k, const void *v, void *k_cache,
                                     float *k_rot_dbg, int B, int Hkv, int T, int d,
                                     const int64_t *k_strides, const int64_t *v_strides,
                                     const int64_t *kc_strides, const yr_rope_table *tab,
                                     void *workspace, size_t workspace_bytes, void *stream) {
    set_error("");
    long long ks[3], vs[3], cs[3];
    int rc = check_prepare(k, v, k_cache, k_rot_dbg, B, Hkv, T, d, k_strides, v_strides,
                           kc_strides, tab, workspace, workspace_bytes, "yr_prefill_prepare_kv",
                           ks, vs, cs);
    if (rc != YR_OK) return rc;
    int sm_count = 0;
    rc = prepare_device(&sm_count);
    if (rc != YR_OK) return rc;
    return launch_prepare(k, v, k_cache, k_rot_dbg, B, Hkv, T, d, ks, vs, cs, tab, workspace,
                          sm_count, static_cast<cudaStream_t>(stream));
}

extern "C" int yr_prefill_attend(const void *q, void *o, float *lse, float *q_rot_dbg, int B,
                                 int Hq, int Hkv, int T, int d, const int64_t *q_strides,
                                 const int64_t *o_strides, const yr_rope_table *tab, int causal,
                                 int window, int n_sink, const void *workspace,
                                 size_t workspace_bytes, void *stream) {
    set_error("");
    long long qs[3], os[3];
    int rc = check_attend(q, o, lse, q_rot_dbg, B, Hq, Hkv, T, d, q_strides, o_strides, tab,
                          causal, window, n_sink, workspace, workspace_bytes, "yr_prefill_attend",
                          qs, os);
    if (rc != YR_OK) return rc;
    rc = prepare_device(nullptr);
    if (rc != YR_OK) return rc;
    return launch_attend(q, o, lse, q_rot_dbg, B, Hq, Hkv, T, d, qs, os, tab, causal, window,
                         n_sink, workspace_planes(workspace, B, Hkv, T, d),
                         static_cast<cudaStream_t>(stream), T, 0);
}

extern "C" int yr_attn_prefill(const void *q, const void *k, const void *v, void *o, float *lse,
                               void *k_cache, float *q_rot_dbg, float *k_rot_dbg, int B, int Hq,
                               int Hkv, int T, int d, const int64_t *q_strides,
                               const int64_t *k_strides, const int64_t *v_strides,
                               const int64_t *o_strides, const int64_t *kc_strides,
                               const yr_rope_table *tab, int causal, int window, int n_sink,
                               void *workspace, size_t workspace_bytes, void *stream) {
    set_error("");
    long long qs[3], os[3], ks[3], vs[3], cs[3];
    int rc = check_attend(q, o, lse, q_rot_dbg, B, Hq, Hkv, T, d, q_strides, o_strides, tab,
                          causal, window, n_sink, workspace, workspace_bytes, "yr_attn_prefill",
                          qs, os);
    if (rc != YR_OK) return rc;
    rc = check_prepare(k, v, k_cache, k_rot_dbg, B, Hkv, T, d, k_strides, v_strides, kc_strides,
                       tab, workspace, workspace_bytes, "yr_attn_prefill", ks, vs, cs);
    if (rc != YR_OK) return rc;
    int sm_count = 0;
    rc = prepare_device(&sm_count);
    if (rc != YR_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = launch_prepare(k, v, k_cache, k_rot_dbg, B, Hkv, T, d, ks, vs, cs, tab, workspace,
                        sm_count, st);
    if (rc != YR_OK) return rc;
    return launch_attend(q, o, lse, q_rot_dbg, B, Hq, Hkv, T, d, qs, os, tab, causal, window,
                         n_sink, workspace_planes(workspace, B, Hkv, T, d), st, T, 0);
}

namespace yr_host {

// The shared body of the two chunked-prefill entry points: argument checks, the
// chunk pass into (k16, v16) with plane stride ld16 starting at slot `first`, then
// the attention over those planes.
// Bytes of one split-KV share's partials: fp32 o [B*Hq*Tq][d] and lse [B*Hq*Tq].
size_t split_share_bytes(long long B, long long Hq, long long Tq, long long d) {
    return static_cast<size_t>(B * Hq * Tq * (d + 1) * 4);
}

// Shares per item for a prefill of Tq query rows after P0 cached keys, when the items
// alone leave SMs idle.  Each CTA holds a whole SM, so the grid runs in waves of
// sm_count CTAs, and a share costs its key tiles plus a CTA's fixed cost (set-up, Q
// rotation, epilogue: about five tiles' time): the count with the least
// waves x (tiles per share + 5) wins.  Each share keeps at least 4 key tiles; at most kMaxSplit shares
// and at most what the split workspace holds.
constexpr int kMaxSplit = 16;
int choose_split(int sm_count, int B, int Hq, int Hkv, int Tq, int P0, int window,
                 size_t ws_bytes, size_t share_bytes) {
    const long long items = attend_items(B, Hq, Hkv, Tq, window);
    if (items >= 2ll * sm_count || share_bytes == 0) return 1;
    const int rows = attend_head_pair(Hq, Hkv, window) ? 128 : 256;  // query rows per CTA
    int keys = P0 + (Tq < rows ? Tq : rows);  // the first query block's keys (the fewest)
    if (window > 0 && window < keys) keys = window + rows;
    const int tiles = (keys + 127) / 128;
    long long s_max = kMaxSplit;
    if (s_max > tiles / 4) s_max = tiles / 4;
    if (s_max > static_cast<long long>(ws_bytes / share_bytes)) s_max = ws_bytes / share_bytes;
    // Time of a split in tile steps: waves x (tiles of a share + the fixed cost).
    int best = 1;
    double best_time = 0.0;
    for (long long s = 1; s <= s_max || s == 1; ++s) {
        const long long waves = (items * s + sm_count - 1) / sm_count;
        const double time = static_cast<double>(waves) *
                            (static_cast<double>(tiles) / static_cast<double>(s) + 5.0);
        if (s == 1 || time < best_time * 0.9999) {
            best_time = time;
            best = static_cast<int>(s);
        }
    }
    return best;
}

int chunk_call(const char *fn, const void *q, const void *k_new, const void *v_new,
               void *k_cache, void *v_cache, void *o, float *lse, int B, int Hq, int Hkv,
               int Tq, int d, int P0, int T_max, const yr_rope_table *tab, int window,
               int n_sink, __half *k16, __half *v16, long long ld16, int first,
               void *split_ws, size_t split_ws_bytes, void *stream) {
    const std::string f(fn);
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !o || !tab)
        return fail(YR_EINVAL, f + ": NULL pointer argument");
    if (B < 1 || Hq < 1 || Hkv < 1 || Tq < 1) return fail(YR_EINVAL, f + ": B, Hq, Hkv and Tq must be >= 1");
    if (P0 < 0 || T_max < 1 || static_cast<long long>(P0) + Tq > T_max)
        return fail(YR_EINVAL, f + ": need 0 <= P0 and P0 + Tq <= T_max");
    const int Tk = P0 + Tq;
    long long qs[3], os[3];
    // check_attend and check_common want a workspace: hand them the fp16 planes, sized
    // for the keys they must hold (the planes' own size is checked by the callers).
    const size_t planes = prefill_ws_bytes(B, Hkv, Tk, d);
    int rc = check_attend(q, o, lse, nullptr, B, Hq, Hkv, Tq, d, nullptr, nullptr, tab, 1, window,
                          n_sink, k16, planes, fn, qs, os);
    if (rc != YR_OK) return rc;
    for (const void *ptr : {k_new, v_new, static_cast<const void *>(k_cache),
                            static_cast<const void *>(v_cache), static_cast<const void *>(v16)})
        if (!aligned(ptr, 16)) return fail(YR_EINVAL, f + ": pointers must be 16-byte aligned");
    int sm_count = 0;
    rc = prepare_device(&sm_count);
    if (rc != YR_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool half = tab->pairs == YR_PAIR_HALF;
    if (Tk > first) {
        yr::ChunkPrepParams cp;
        std::memset(&cp, 0, sizeof cp);
        cp.k_new = static_cast<const __nv_bfloat16 *>(k_new);
        cp.v_new = static_cast<const __nv_bfloat16 *>(v_new);
        cp.kc = static_cast<__nv_bfloat16 *>(k_cache);
        cp.vc = static_cast<__nv_bfloat16 *>(v_cache);
        cp.k16 = k16;
        cp.v16 = v16;
        cp.Tq = Tq; cp.P0 = P0; cp.Tk = Tk; cp.T_max = T_max; cp.d = d;
        cp.first = first;
        cp.ld16 = ld16;
        cp.n_items = static_cast<long long>(B) * Hkv * (Tk - first) * (half ? d / 16 : d / 8);
        for (int i = 0; i < d / 2; ++i) cp.turns[i] = tab->turns[i];
        long long blocks = (cp.n_items + 255) / 256;
        const long long cap = static_cast<long long>(sm_count) * 16;
        if (blocks > cap) blocks = cap;
        if (half)
            yr::chunk_prep_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(cp);
        else
            yr::chunk_prep_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(cp);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("chunk_prep_kernel launch", e);
    }
    const size_t share = split_share_bytes(B, Hq, Tq, d);
    const int n_split = split_ws ? choose_split(sm_count, B, Hq, Hkv, Tq, P0, window, split_ws_bytes,
                                                share)
                                 : 1;
    const KvPlanes kv{k16, v16, ld16};
    if (n_split == 1)
        return launch_attend(q, o, lse, nullptr, B, Hq, Hkv, Tq, d, qs, os, tab, 1, window,
                             n_sink, kv, st, Tk, P0);
    // Split-KV: the shares' fp32 partials, then their log-sum-exp merge into o.
    const long long rows = static_cast<long long>(B) * Hq * Tq;
    float *o_part = static_cast<float *>(split_ws);
    float *lse_part = o_part + n_split * rows * d;
    rc = launch_attend(q, nullptr, lse_part, nullptr, B, Hq, Hkv, Tq, d, qs, os, tab, 1, window,
                       n_sink, kv, st, Tk, P0, 0, o_part, n_split);
    if (rc != YR_OK) return rc;
    yr::SplitMergeParams mp;
    mp.o_part = o_part;
    mp.lse_part = lse_part;
    mp.o = static_cast<__nv_bfloat16 *>(o);
    mp.lse = lse;
    mp.rows = rows;
    mp.d = d;
    mp.n_split = n_split;
    long long blocks = (rows * (d / 8) + 255) / 256;
    const long long cap = static_cast<long long>(sm_count) * 16;
    if (blocks > cap) blocks = cap;
    yr::split_merge_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(mp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("split_merge_kernel launch", e);
    return YR_OK;
}

}  // namespace yr_host

extern "C" int yr_attn_prefill_chunk(const void *q, const void *k_new, const void *v_new,
                                     void *k_cache, void *v_cache, void *o, float *lse, int B,
                                     int Hq, int Hkv, int Tq, int d, int P0, int T_max,
                                     const yr_rope_table *tab, int window, int n_sink,
                                     void *workspace, size_t workspace_bytes, void *stream) {
    set_error("");
    const char *fn = "yr_attn_prefill_chunk";
    if (!workspace) return fail(YR_EINVAL, std::string(fn) + ": workspace must be non-NULL");
    if (B < 1 || Hkv < 1 || Tq < 1 || P0 < 0 || static_cast<long long>(P0) + Tq > (1ll << 30))
        return fail(YR_EINVAL, std::string(fn) + ": B, Hkv, Tq >= 1 and 0 <= P0 needed");
    const int Tk = P0 + Tq;
    const size_t need = prefill_ws_bytes(B, Hkv, Tk, d);
    if (workspace_bytes < need)
        return fail(YR_EINVAL, std::string(fn) + ": workspace too small (need " +
                                   std::to_string(need) + " bytes)");
    if (!aligned(workspace, 256))
        return fail(YR_EINVAL, std::string(fn) + ": workspace must be 256-byte aligned");
    const KvPlanes kv = workspace_planes(workspace, B, Hkv, Tk, d);
    return chunk_call(fn, q, k_new, v_new, k_cache, v_cache, o, lse, B, Hq, Hkv, Tq, d, P0,
                      T_max, tab, window, n_sink, const_cast<__half *>(kv.k16),
                      const_cast<__half *>(kv.v16), Tk, 0, nullptr, 0, stream);
}

extern "C" size_t yr_attn_prefill_chunk_split_bytes(int B, int Hq, int Tq, int d) {
    if (B < 1 || Hq < 1 || Tq < 1 || (d != 64 && d != 128)) return 0;
    return kMaxSplit * split_share_bytes(B, Hq, Tq, d);
}

extern "C" int yr_attn_prefill_chunk_fp16cache(const void *q, const void *k_new,
                                               const void *v_new, void *k_cache, void *v_cache,
                                               void *k_cache16, void *v_cache16, int cache16_len,
                                               void *o, float *lse, int B, int Hq, int Hkv,
                                               int Tq, int d, int P0, int T_max,
                                               const yr_rope_table *tab, int window, int n_sink,
                                               void *workspace, size_t workspace_bytes,
                                               void *stream) {
    set_error("");
    const char *fn = "yr_attn_prefill_chunk_fp16cache";
    if (!k_cache16 || !v_cache16)
        return fail(YR_EINVAL, std::string(fn) + ": k_cache16 and v_cache16 must be non-NULL");
    if (!aligned(k_cache16, 256) || !aligned(v_cache16, 256))
        return fail(YR_EINVAL, std::string(fn) + ": the fp16 caches must be 256-byte aligned");
    if (cache16_len < 0 || cache16_len > P0)
        return fail(YR_EINVAL, std::string(fn) + ": need 0 <= cache16_len <= P0");
    if (workspace && !aligned(workspace, 256))
        return fail(YR_EINVAL, std::string(fn) + ": workspace must be 256-byte aligned");
    return chunk_call(fn, q, k_new, v_new, k_cache, v_cache, o, lse, B, Hq, Hkv, Tq, d, P0,
                      T_max, tab, window, n_sink, static_cast<__half *>(k_cache16),
                      static_cast<__half *>(v_cache16), T_max, cache16_len, workspace,
                      workspace ? workspace_bytes : 0, stream);
}

extern "C" int yr_prefill_prepare_kv_at(const void *k, const void *v, void *k_cache,
                                        float *k_rot_dbg, int B, int Hkv, int T, int d,
                                        const int64_t *k_strides, const int64_t *v_strides,
                                        const int64_t *kc_strides, const yr_rope_table *tab,
                                        int k_pos0, void *workspace, size_t workspace_bytes,
                                        void *stream) {
    set_error("");
    if (k_pos0 < 0 || static_cast<long long>(k_pos0) + T > (1ll << 30))
        return fail(YR_EINVAL, "yr_prefill_prepare_kv_at: need 0 <= k_pos0 and k_pos0 + T <= 2^30");
    long long ks[3], vs[3], cs[3];
    int rc = check_prepare(k, v, k_cache, k_rot_dbg, B, Hkv, T, d, k_strides, v_strides,
                           kc_strides, tab, workspace, workspace_bytes, "yr_prefill_prepare_kv_at",
                           ks, vs, cs);
    if (rc != YR_OK) return rc;
    int sm_count = 0;
    rc = prepare_device(&sm_count);
    if (rc != YR_OK) return rc;
    return launch_prepare(k, v, k_cache, k_rot_dbg, B, Hkv, T, d, ks, vs, cs, tab, workspace,
                          sm_count, static_cast<cudaStream_t>(stream), k_pos0);
}

extern "C" int yr_prefill_attend_block(const void *q, float *o, float *lse, int B, int Hq,
                                       int Hkv, int T, int Tk, int d, const int64_t *q_strides,
                                       const yr_rope_table *tab, int causal, int window,
                                       int n_sink, int q_pos0, int k_pos0, const void *workspace,
                                       size_t workspace_bytes, void *stream) {
    set_error("");
    const std::string f("yr_prefill_attend_block");
    if (Tk < 1) return fail(YR_EINVAL, f + ": Tk must be >= 1");
    if (q_pos0 < 0 || k_pos0 < 0 || static_cast<long long>(q_pos0) + T > (1ll << 30) ||
        static_cast<long long>(k_pos0) + Tk > (1ll << 30))
        return fail(YR_EINVAL, f + ": positions must be >= 0 and end below 2^30");
    if (causal && q_pos0 < k_pos0)
        return fail(YR_EINVAL, f + ": causal blocks need q_pos0 >= k_pos0 (a block wholly in the "
                                   "future has no visible key; skip it)");
    long long qs[3], os[3];
    // o is fp32 and contiguous here; check_attend's bf16 stride checks see it as such.
    int rc = check_attend(q, o, lse, nullptr, B, Hq, Hkv, T, d, q_strides, nullptr, tab, causal,
                          window, n_sink, workspace, workspace_bytes, f.c_str(), qs, os);
    if (rc != YR_OK) return rc;
    rc = check_common(f.c_str(), B, Hkv, Tk, d, tab, workspace, workspace_bytes);
    if (rc != YR_OK) return rc;
    rc = prepare_device(nullptr);
    if (rc != YR_OK) return rc;
    // Sinks are the first n_sink positions of the whole sequence: in this block's key
    // coordinates they are keys [0, n_sink - k_pos0).
    const int sinks_here = n_sink > k_pos0 ? n_sink - k_pos0 : 0;
    return launch_attend(q, nullptr, lse, nullptr, B, Hq, Hkv, T, d, qs, os, tab, causal, window,
                         sinks_here, workspace_planes(workspace, B, Hkv, Tk, d),
                         static_cast<cudaStream_t>(stream), Tk, q_pos0 - k_pos0, k_pos0, o);
}

extern "C" int yr_attn_merge(const float *o_part, const float *lse_part, float *o_acc,
                             float *lse_acc, void *o_out, long long rows, int d, int init,
                             void *stream) {
    set_error("");
    const std::string f("yr_attn_merge");
    if (!o_part || !lse_part || !o_acc || !lse_acc)
        return fail(YR_EINVAL, f + ": o_part, lse_part, o_acc and lse_acc must be non-NULL");
    if (rows < 1) return fail(YR_EINVAL, f + ": rows must be >= 1");
    if (d != 64 && d != 128) return fail(YR_EUNSUPPORTED, f + ": d must be 64 or 128");
    for (const void *ptr : {static_cast<const void *>(o_part), static_cast<const void *>(o_acc),
                            static_cast<const void *>(o_out)})
        if (ptr && !aligned(ptr, 16)) return fail(YR_EINVAL, f + ": o pointers must be 16-byte aligned");
    if (!aligned(lse_part, 4) || !aligned(lse_acc, 4))
        return fail(YR_EINVAL, f + ": lse pointers must be 4-byte aligned");
    int sm_count = 0;
    int rc = prepare_device(&sm_count);
    if (rc != YR_OK) return rc;
    yr::MergeParams mp;
    mp.o_part = o_part;
    mp.lse_part = lse_part;
    mp.o_acc = o_acc;
    mp.lse_acc = lse_acc;
    mp.o_out = static_cast<__nv_bfloat16 *>(o_out);
    mp.rows = rows;
    mp.d = d;
    mp.init = init ? 1 : 0;
    const long long rows_per_block = 8LL * (32 / (d / 8));  // 8 warps
    long long blocks = (rows + rows_per_block - 1) / rows_per_block;
    const long long cap = static_cast<long long>(sm_count) * 16;
    if (blocks > cap) blocks = cap;
    yr::attn_merge_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                            static_cast<cudaStream_t>(stream)>>>(mp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("attn_merge_kernel launch", e);
    return YR_OK;
}

extern "C" int yr_attn_decode(const void *q_new, const void *k_new, const void *v_new,
                              void *k_cache, void *v_cache, const int32_t *cache_len, void *o,
                              float *lse, float *q_rot_dbg, int B, int Hq, int Hkv, int d,
                              int T_max, const yr_rope_table *tab, int window, int n_sink,
                              void *workspace, size_t workspace_bytes, void *stream) {
    set_error("");
    if (!q_new || !k_new || !v_new || !k_cache || !v_cache || !cache_len || !o || !tab || !workspace)
        return fail(YR_EINVAL, "yr_attn_decode: NULL pointer argument");
    if (B < 1 || Hq < 1 || Hkv < 1 || T_max < 1)
        return fail(YR_EINVAL, "yr_attn_decode: B, Hq, Hkv and T_max must be >= 1");
    if (Hq % Hkv != 0) return fail(YR_EINVAL, "yr_attn_decode: Hq must be a multiple of Hkv");
    if (d != 64 && d != 128) return fail(YR_EUNSUPPORTED, "yr_attn_decode: d must be 64 or 128");
    if (Hq / Hkv > 16) return fail(YR_EUNSUPPORTED, "yr_attn_decode: at most 16 query heads per KV head");
    if (tab->head_dim != d) return fail(YR_EINVAL, "yr_attn_decode: table head_dim != d");
    if (tab->pairs != YR_PAIR_INTERLEAVED && tab->pairs != YR_PAIR_HALF)
        return fail(YR_EINVAL, "yr_attn_decode: table pairs must be YR_PAIR_INTERLEAVED or YR_PAIR_HALF");
    if (window < 0 || n_sink < 0) return fail(YR_EINVAL, "yr_attn_decode: window and n_sink must be >= 0");
    if (n_sink > 0 && window == 0) return fail(YR_EINVAL, "yr_attn_decode: sinks need a window");
    const size_t need = decode_ws_bytes(B, Hq, Hkv, d, T_max);
    if (workspace_bytes < need)
        return fail(YR_EINVAL, "yr_attn_decode: workspace too small (need " + std::to_string(need) + " bytes)");
    if (!aligned(workspace, 256)) return fail(YR_EINVAL, "yr_attn_decode: workspace must be 256-byte aligned");
    for (const void *ptr : {q_new, k_new, v_new, static_cast<const void *>(k_cache),
                            static_cast<const void *>(v_cache), static_cast<const void *>(o)})
        if (!aligned(ptr, 16)) return fail(YR_EINVAL, "yr_attn_decode: tensor pointers must be 16-byte aligned");
    if (!aligned(cache_len, 4) || (lse && !aligned(lse, 4)) || (q_rot_dbg && !aligned(q_rot_dbg, 4)))
        return fail(YR_EINVAL, "yr_attn_decode: cache_len/lse/q_rot_dbg must be 4-byte aligned");
    int sm_count = 0;
    int rc = prepare_device(&sm_count);
    if (rc != YR_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int g = Hq / Hkv;
    const int nc = decode_parts(T_max);
    yr::DecodeParams dp;
    std::memset(&dp, 0, sizeof dp);
    dp.q_new = static_cast<const __nv_bfloat16 *>(q_new);
    dp.k_new = static_cast<const __nv_bfloat16 *>(k_new);
    dp.v_new = static_cast<const __nv_bfloat16 *>(v_new);
    dp.k_cache = static_cast<__nv_bfloat16 *>(k_cache);
    dp.v_cache = static_cast<__nv_bfloat16 *>(v_cache);
    dp.cache_len = cache_len;
    dp.ws_o = static_cast<float *>(workspace);
    dp.ws_ml = dp.ws_o + static_cast<size_t>(B) * Hkv * nc * g * d;
    dp.o = static_cast<__nv_bfloat16 *>(o);
    dp.lse = lse;
    dp.q_dbg = q_rot_dbg;
    dp.B = B; dp.Hq = Hq; dp.Hkv = Hkv; dp.T_max = T_max; dp.group = g; dp.n_parts = nc;
    dp.window = window; dp.n_sink = n_sink;
    dp.sl2 = static_cast<float>(tab->softmax_scale * 1.4426950408889634);
    dp.alibi = tab->method == YR_ALIBI ? 1 : 0;
    dp.half_pairs = tab->pairs == YR_PAIR_HALF ? 1 : 0;
    for (int i = 0; i < d / 2; ++i) dp.turns[i] = tab->turns[i];
    if (d == 128) {
        if (g <= 8) {
            dp.grid_blocks = decode_grid<128, 1>(sm_count);
            yr::decode_split_kernel<128, 1><<<dp.grid_blocks, yr::kDecThreads, yr::decode_smem_bytes<128>(), st>>>(dp);
        } else {
            dp.grid_blocks = decode_grid<128, 2>(sm_count);
            yr::decode_split_kernel<128, 2><<<dp.grid_blocks, yr::kDecThreads, yr::decode_smem_bytes<128>(), st>>>(dp);
        }
    } else {
        if (g <= 8) {
            dp.grid_blocks = decode_grid<64, 1>(sm_count);
            yr::decode_split_kernel<64, 1><<<dp.grid_blocks, yr::kDecThreads, yr::decode_smem_bytes<64>(), st>>>(dp);
        } else {
            dp.grid_blocks = decode_grid<64, 2>(sm_count);
            yr::decode_split_kernel<64, 2><<<dp.grid_blocks, yr::kDecThreads, yr::decode_smem_bytes<64>(), st>>>(dp);
        }
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("decode_split_kernel launch", e);
    const dim3 mgrid(Hq, B);
    if (d == 128)
        yr::decode_merge_kernel<128><<<mgrid, 128, 0, st>>>(dp);
    else
        yr::decode_merge_kernel<64><<<mgrid, 64, 0, st>>>(dp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("decode_merge_kernel launch", e);
    return YR_OK;
}

// ------------------------------------------------------------------------------
// Decode without a caller-supplied workspace.  The split-KV partial results go to
// this fixed array instead; every GPU that loads the library holds it until exit.
// In host code `g_decode_noalloc_scratch` is only a stand-in for the symbol, not a
// device address: the address is looked up per context with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[YR_DECODE_NOALLOC_SCRATCH_BYTES];

namespace yr_host {
std::mutex g_scratch_mu;
std::unordered_map<unsigned long long, void *> g_scratch_ptr;  // by context id

// Set-up, once per context (each device's primary context, or a context the host
// application made current), with that context current: the address of the array
// in the context's instance of this module.
int noalloc_scratch(void **out) {
    int dev = 0;
    unsigned long long ctx = 0;
    int rc = current_context(&dev, &ctx);
    if (rc != YR_OK) return rc;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    auto it = g_scratch_ptr.find(ctx);
    if (it == g_scratch_ptr.end()) {
        void *ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_decode_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress(decode scratch)", e);
        it = g_scratch_ptr.emplace(ctx, ptr).first;
    }
    *out = it->second;
    return YR_OK;
}
}  // namespace yr_host

extern "C" int yr_attn_decode_noalloc(const void *q_new, const void *k_new, const void *v_new,
                                      void *k_cache, void *v_cache, const int32_t *cache_len,
                                      void *o, float *lse, float *q_rot_dbg, int B, int Hq,
                                      int Hkv, int d, int T_max, const yr_rope_table *tab,
                                      int window, int n_sink, void *stream) {
    set_error("");
    const size_t need = yr_attn_decode_workspace_bytes(B, Hq, Hkv, d, T_max);
    if (need == 0)
        return fail(YR_EINVAL, "yr_attn_decode_noalloc: invalid sizes (B, Hq, Hkv, d, T_max)");
    if (need > static_cast<size_t>(YR_DECODE_NOALLOC_SCRATCH_BYTES))
        return fail(YR_EINVAL, "yr_attn_decode_noalloc: this call needs " + std::to_string(need) +
                                   " bytes of scratch, more than the fixed " +
                                   std::to_string(YR_DECODE_NOALLOC_SCRATCH_BYTES) +
                                   " bytes; use yr_attn_decode with a workspace");
    void *scratch = nullptr;
    int rc = noalloc_scratch(&scratch);
    if (rc != YR_OK) return rc;
    rc = yr_attn_decode(q_new, k_new, v_new, k_cache, v_cache, cache_len, o, lse, q_rot_dbg, B,
                        Hq, Hkv, d, T_max, tab, window, n_sink, scratch,
                        YR_DECODE_NOALLOC_SCRATCH_BYTES, stream);
    if (rc != YR_OK) {
        std::string m = g_err;
        if (m.rfind("yr_attn_decode:", 0) == 0) m = "yr_attn_decode_noalloc:" + m.substr(15);
        set_error(m);
    }
    return rc;
}

extern "C" int yr_device_status(void *stream) {
    set_error("");
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail("cudaStreamSynchronize", e);
    unsigned v = 0;
    e = cudaMemcpyFromSymbol(&v, g_yr_status, sizeof v);
    if (e != cudaSuccess) return cuda_fail("reading the status word", e);
    if (v == 0) return YR_OK;
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_yr_status, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail("clearing the status word", e);
    std::string msg = "device status:";
    if (v & yr::kStatusTimeoutLoad) msg += " prefill-load-timeout";
    if (v & yr::kStatusTimeoutMma) msg += " prefill-mma-timeout";
    if (v & yr::kStatusTimeoutSoftmax) msg += " prefill-softmax-timeout";
    if (v & yr::kStatusTimeoutDrain) msg += " prefill-drain-timeout";
    if (v & yr::kStatusBadCacheLen) msg += " decode-cache-length-out-of-range";
    if (v & yr::kStatusRange)
        msg += " prefill-operand-outside-fp16-range (|rotated q|, |rotated k| or |v| >= 65520,"
               " or not a number)";
    set_error(msg);
    if (v & 0xFFu) return YR_ETIMEOUT;
    return (v & yr::kStatusRange) ? YR_ERANGE : YR_EINVAL;
}
