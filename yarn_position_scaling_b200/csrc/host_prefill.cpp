// host_prefill.cpp -- prefill of prompts that live in host memory: the host-to-device
// copies of q, k and v, the rotated-key pass and attention, and the device-to-host copy
// of the output, cut into (batch, KV-head group) units and overlapped on three streams
// so that the PCIe transfers of some units run while others compute.
//
// A plan owns two streams (copy-in, copy-out) and one event per unit and stage; the
// caller owns the device workspace it carves its buffers from.  Unit u's copy-in of a
// call waits only for the previous call's kernels on unit u (its input buffers are
// free then), and its kernels only for the previous call's copy-out of unit u, so
// successive calls overlap unit by unit as well.  The kernels run on the caller's
// stream through yr_attn_prefill; the caller's stream also waits for the last
// copy-out before its later work.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "../../include/yarnattn.h"

namespace yr_host {
void set_error(const std::string &msg);
}

namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Layout {
    size_t q_bytes, kv_bytes, ws_bytes, total;
    int kv_per_unit;
};

// Device buffers of a plan: q, k, v and o for the whole shape, then one prefill
// workspace for a unit's KV heads (the units' kernels run one after another).
bool layout(int B, int Hq, int Hkv, int T, int d, int units_per_batch, Layout *out) {
    if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || (d != 64 && d != 128) || Hq % Hkv) return false;
    int n = units_per_batch > 0 ? units_per_batch : (Hkv < 8 ? Hkv : 8);
    if (n > Hkv) n = Hkv;
    out->kv_per_unit = (Hkv + n - 1) / n;
    out->q_bytes = static_cast<size_t>(B) * Hq * T * d * 2;
    out->kv_bytes = static_cast<size_t>(B) * Hkv * T * d * 2;
    out->ws_bytes = yr_attn_prefill_workspace_bytes(1, out->kv_per_unit, T, d);
    out->total = 2 * round_up(out->q_bytes) + 2 * round_up(out->kv_bytes) + round_up(out->ws_bytes);
    return true;
}

int fail(int code, const std::string &msg) {
    yr_host::set_error(msg);
    return code;
}

int cuda_fail(const char *what, cudaError_t e) {
    return fail(YR_ECUDA, std::string("yr_host_prefill: ") + what + ": " + cudaGetErrorString(e));
}

}  // namespace

struct yr_host_prefill {
    int B, Hq, Hkv, T, d, group, device;
    Layout lay;
    char *qd, *kd, *vd, *od, *ws;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    struct Unit {
        int b, kv0, kv1;
        cudaEvent_t arrived = nullptr, computed = nullptr, copied_out = nullptr;
        // recorded by an earlier call (kept per unit, so that a call that stopped on an
        // error half-way still orders the next call behind the work it did queue)
        bool has_computed = false, has_copied_out = false;
    };
    std::vector<Unit> units;
    cudaEvent_t all_out = nullptr;
};

namespace {

void release(yr_host_prefill *p) {
    for (auto &u : p->units)
        for (cudaEvent_t e : {u.arrived, u.computed, u.copied_out})
            if (e) cudaEventDestroy(e);
    if (p->all_out) cudaEventDestroy(p->all_out);
    if (p->h2d) cudaStreamDestroy(p->h2d);
    if (p->d2h) cudaStreamDestroy(p->d2h);
    delete p;
}

}  // namespace

extern "C" size_t yr_host_prefill_workspace_bytes(int B, int Hq, int Hkv, int T, int d,
                                                  int units_per_batch) {
    Layout l;
    return layout(B, Hq, Hkv, T, d, units_per_batch, &l) ? l.total : 0;
}

extern "C" int yr_host_prefill_create(yr_host_prefill **plan, int B, int Hq, int Hkv, int T,
                                      int d, int units_per_batch, void *workspace,
                                      size_t workspace_bytes) {
    yr_host::set_error("");
    if (!plan || !workspace) return fail(YR_EINVAL, "yr_host_prefill_create: NULL argument");
    *plan = nullptr;
    Layout lay;
    if (!layout(B, Hq, Hkv, T, d, units_per_batch, &lay))
        return fail(YR_EINVAL, "yr_host_prefill_create: invalid sizes (B, Hq, Hkv, T >= 1, "
                               "Hq a multiple of Hkv, d 64 or 128)");
    if (workspace_bytes < lay.total)
        return fail(YR_EINVAL, "yr_host_prefill_create: workspace too small (need " +
                                   std::to_string(lay.total) + " bytes)");
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign)
        return fail(YR_EINVAL, "yr_host_prefill_create: workspace must be 256-byte aligned");
    auto *p = new (std::nothrow) yr_host_prefill();
    if (!p) return fail(YR_ECUDA, "yr_host_prefill_create: out of host memory");
    p->B = B; p->Hq = Hq; p->Hkv = Hkv; p->T = T; p->d = d; p->group = Hq / Hkv;
    p->lay = lay;
    char *base = static_cast<char *>(workspace);
    p->qd = base;
    p->kd = p->qd + round_up(lay.q_bytes);
    p->vd = p->kd + round_up(lay.kv_bytes);
    p->od = p->vd + round_up(lay.kv_bytes);
    p->ws = p->od + round_up(lay.q_bytes);
    cudaError_t e = cudaGetDevice(&p->device);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->d2h, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->all_out, cudaEventDisableTiming);
    for (int b = 0; b < B && e == cudaSuccess; ++b)
        for (int kv0 = 0; kv0 < Hkv && e == cudaSuccess; kv0 += lay.kv_per_unit) {
            yr_host_prefill::Unit u;
            u.b = b;
            u.kv0 = kv0;
            u.kv1 = kv0 + lay.kv_per_unit < Hkv ? kv0 + lay.kv_per_unit : Hkv;
            e = cudaEventCreateWithFlags(&u.arrived, cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&u.computed, cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&u.copied_out, cudaEventDisableTiming);
            p->units.push_back(u);
        }
    if (e != cudaSuccess) {
        release(p);
        return cuda_fail("creating streams and events", e);
    }
    *plan = p;
    return YR_OK;
}

extern "C" int yr_host_prefill_run(yr_host_prefill *p, const void *q, const void *k,
                                   const void *v, void *o, const yr_rope_table *tab, int causal,
                                   int window, int n_sink, void *stream) {
    yr_host::set_error("");
    if (!p || !q || !k || !v || !o || !tab)
        return fail(YR_EINVAL, "yr_host_prefill_run: NULL argument");
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (dev != p->device)
        return fail(YR_EINVAL, "yr_host_prefill_run: the plan belongs to another device");
    cudaStream_t comp = static_cast<cudaStream_t>(stream);
    const size_t row = static_cast<size_t>(p->T) * p->d * 2;  // bytes of one head's rows
    const size_t ws_bytes = p->lay.ws_bytes;
    for (auto &u : p->units) {
        const int nkv = u.kv1 - u.kv0;
        const size_t q_off = (static_cast<size_t>(u.b) * p->Hq + static_cast<size_t>(u.kv0) * p->group) * row;
        const size_t q_len = static_cast<size_t>(nkv) * p->group * row;
        const size_t kv_off = (static_cast<size_t>(u.b) * p->Hkv + u.kv0) * row;
        const size_t kv_len = static_cast<size_t>(nkv) * row;
        // copy-in: once the previous call's kernels on this unit have read its inputs
        if (u.has_computed && (e = cudaStreamWaitEvent(p->h2d, u.computed, 0)) != cudaSuccess)
            return cuda_fail("cudaStreamWaitEvent", e);
        if ((e = cudaMemcpyAsync(p->qd + q_off, static_cast<const char *>(q) + q_off, q_len,
                                 cudaMemcpyHostToDevice, p->h2d)) != cudaSuccess ||
            (e = cudaMemcpyAsync(p->kd + kv_off, static_cast<const char *>(k) + kv_off, kv_len,
                                 cudaMemcpyHostToDevice, p->h2d)) != cudaSuccess ||
            (e = cudaMemcpyAsync(p->vd + kv_off, static_cast<const char *>(v) + kv_off, kv_len,
                                 cudaMemcpyHostToDevice, p->h2d)) != cudaSuccess ||
            (e = cudaEventRecord(u.arrived, p->h2d)) != cudaSuccess)
            return cuda_fail("copy-in", e);
        // kernels: once the inputs have arrived and the previous output has left
        if ((e = cudaStreamWaitEvent(comp, u.arrived, 0)) != cudaSuccess ||
            (u.has_copied_out && (e = cudaStreamWaitEvent(comp, u.copied_out, 0)) != cudaSuccess))
            return cuda_fail("cudaStreamWaitEvent", e);
        const int rc = yr_attn_prefill(p->qd + q_off, p->kd + kv_off, p->vd + kv_off,
                                       p->od + q_off, nullptr, nullptr, nullptr, nullptr, 1,
                                       nkv * p->group, nkv, p->T, p->d, nullptr, nullptr,
                                       nullptr, nullptr, nullptr, tab, causal, window, n_sink,
                                       p->ws, ws_bytes, comp);
        if (rc != YR_OK) return rc;  // its message is already set
        if ((e = cudaEventRecord(u.computed, comp)) != cudaSuccess)
            return cuda_fail("cudaEventRecord", e);
        u.has_computed = true;
        // copy-out
        if ((e = cudaStreamWaitEvent(p->d2h, u.computed, 0)) != cudaSuccess ||
            (e = cudaMemcpyAsync(static_cast<char *>(o) + q_off, p->od + q_off, q_len,
                                 cudaMemcpyDeviceToHost, p->d2h)) != cudaSuccess ||
            (e = cudaEventRecord(u.copied_out, p->d2h)) != cudaSuccess)
            return cuda_fail("copy-out", e);
        u.has_copied_out = true;
    }
    if ((e = cudaEventRecord(p->all_out, p->d2h)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(comp, p->all_out, 0)) != cudaSuccess)
        return cuda_fail("joining the caller's stream", e);
    return YR_OK;
}

extern "C" int yr_host_prefill_destroy(yr_host_prefill *p) {
    yr_host::set_error("");
    if (!p) return YR_OK;
    cudaError_t e = cudaStreamSynchronize(p->h2d);
    if (e == cudaSuccess) e = cudaStreamSynchronize(p->d2h);
    release(p);
    return e == cudaSuccess ? YR_OK : cuda_fail("cudaStreamSynchronize", e);
}
