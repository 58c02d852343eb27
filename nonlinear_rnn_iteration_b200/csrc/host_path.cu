// host_path.cu -- the Newton forward on host buffers, copies overlapped with
// the solve.
//
// A serving caller usually holds the pre-activations in host memory and
// wants H back there.  Copying everything in, solving, and copying
// everything out leaves the PCIe link idle in one direction at a time and
// the GPU idle during both copies.  Batch rows are independent recurrences
// (the tiles of the solver never span two rows), so this entry point cuts
// the batch into slices of rows and pipelines them through kSlots device
// slots on three streams -- copy in, solve, copy out -- so that slice i+1
// comes in while slice i is solved and slice i-1 goes out.  Every row's
// result is bit-identical to what pararnn_newton_forward returns for the
// whole batch.  The channels are independent recurrences too, so a slice
// may also take only a range of channels (copied with strided 2-D copies):
// more, smaller slices shorten the pipeline's fill and drain, when only the
// first slice's copy in and the last one's solve and copy out run alone.
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "pararnn_b200.h"

namespace pararnn {
pararnn_status newton_forward_slice(int64_t B_whole, int64_t D_whole, pararnn_cell cell, int64_t B, int64_t T,
                                    int64_t D, pararnn_dtype px_dtype, const void* preacts, const float* diag_w,
                                    const float* h0, int K, float* H_out, void* workspace, size_t ws_bytes,
                                    void* stream);  // pararnn_abi.cu
void set_last_error(const char* msg);   // pararnn_abi.cu
bool pointer_on_device(const void* p);  // pararnn_abi.cu

namespace hp {

constexpr int kSlots = 3;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Layout {
    int64_t rows = 0;   // batch rows per slice
    int64_t chans = 0;  // channels per slice
    size_t px_bytes = 0, h_bytes = 0, w_bytes = 0, h0_bytes = 0, fw_bytes = 0, slot_bytes = 0, total = 0;
};

// channels_per_slice: 0 (or >= D) for whole rows, else a multiple of 8 with
// D a multiple of 8, so that every slice's rows keep the 16-byte alignment
// the whole batch has and the solver takes the same path (bit-identical
// results)
bool layout(pararnn_cell cell, int64_t B, int64_t T, int64_t D, int K, int64_t rows_per_slice,
            int64_t channels_per_slice, size_t esz, Layout& l) {
    const int G = pararnn_num_gates(cell), S = pararnn_state_width(cell);
    if (G < 0 || B < 0 || T < 0 || D < 0 || rows_per_slice < 1 || channels_per_slice < 0) return false;
    const bool split = channels_per_slice > 0 && channels_per_slice < D;
    if (split && (channels_per_slice % 8 != 0 || D % 8 != 0)) return false;
    l.rows = rows_per_slice < B ? rows_per_slice : (B > 0 ? B : 1);
    l.chans = split ? channels_per_slice : (D > 0 ? D : 1);
    l.fw_bytes = pararnn_workspace_bytes(cell, l.rows, T, l.chans, K);
    if (l.fw_bytes == 0) return false;
    l.px_bytes = align256((size_t)l.rows * T * G * l.chans * esz);
    l.h_bytes = align256((size_t)l.rows * T * S * l.chans * sizeof(float));
    // a channel slice's own copies of the weights and of h0 (contiguous)
    l.w_bytes = split ? align256((size_t)G * l.chans * sizeof(float)) : 0;
    l.h0_bytes = split ? align256((size_t)l.rows * S * l.chans * sizeof(float)) : 0;
    l.slot_bytes = align256(l.fw_bytes) + l.px_bytes + l.h_bytes + l.w_bytes + l.h0_bytes;
    l.total = 256 + kSlots * l.slot_bytes;
    return true;
}

// fold one slot's device status into the call's header.  A forward on the
// small-problem path leaves its flags in the tagged word (header bytes 8..15,
// valid when their tag equals the call number at bytes 16..19); every other
// forward clears those bytes and uses word 0.
__global__ void fold_status(unsigned* dst, const unsigned* src) {
    if (threadIdx.x != 0) return;
    unsigned f = src[0];
    const unsigned ep = src[4];
    if (ep) {
        const unsigned long long tw = *reinterpret_cast<const unsigned long long*>(src + 2);
        f = (static_cast<unsigned>(tw >> 32) == ep) ? static_cast<unsigned>(tw) : 0u;
    }
    if (f) atomicOr(dst, f);
}

pararnn_status fail(pararnn_status st, const char* msg) {
    set_last_error(msg);
    return st;
}

}  // namespace hp
}  // namespace pararnn

using namespace pararnn;

extern "C" size_t pararnn_newton_forward_host_workspace_bytes(pararnn_cell cell, int64_t B, int64_t T, int64_t D,
                                                              int K, pararnn_dtype px_dtype, int64_t rows_per_slice,
                                                              int64_t channels_per_slice) {
    hp::Layout l;
    const size_t esz = px_dtype == PARARNN_BF16 ? 2 : 4;
    if (px_dtype != PARARNN_F32 && px_dtype != PARARNN_BF16) return 0;
    if (!hp::layout(cell, B, T, D, K, rows_per_slice, channels_per_slice, esz, l)) return 0;
    return l.total;
}

extern "C" pararnn_status pararnn_newton_forward_host(pararnn_cell cell, int64_t B, int64_t T, int64_t D,
                                                      pararnn_dtype px_dtype, const void* preacts_host,
                                                      const float* diag_w, const float* h0, int K, float* H_host,
                                                      void* workspace, size_t ws_bytes, int64_t rows_per_slice,
                                                      int64_t channels_per_slice, void* stream) {
    if (px_dtype != PARARNN_F32 && px_dtype != PARARNN_BF16)
        return hp::fail(PARARNN_EINVAL, "pararnn_newton_forward_host: unknown pre-activation dtype");
    const size_t esz = px_dtype == PARARNN_BF16 ? 2 : 4;
    hp::Layout l;
    if (!hp::layout(cell, B, T, D, K, rows_per_slice, channels_per_slice, esz, l))
        return hp::fail(PARARNN_EINVAL, "pararnn_newton_forward_host: bad cell, sizes, K, rows_per_slice or "
                                        "channels_per_slice");
    if (!workspace || ws_bytes < l.total || !pointer_on_device(workspace) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255))
        return hp::fail(PARARNN_EINVAL, "pararnn_newton_forward_host: workspace missing, small or not 256-byte "
                                        "aligned device memory (see pararnn_newton_forward_host_workspace_bytes)");
    cudaStream_t user = static_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    cudaError_t e = cudaMemsetAsync(ws, 0, 256, user);
    if (e != cudaSuccess) return hp::fail(PARARNN_ECUDA, "pararnn_newton_forward_host: header reset failed");
    if (B == 0 || T == 0 || D == 0) return PARARNN_OK;
    if (!preacts_host || !H_host)
        return hp::fail(PARARNN_EINVAL, "pararnn_newton_forward_host: preacts_host and H_host are required");
    const int G = pararnn_num_gates(cell), S = pararnn_state_width(cell);
    const int64_t nrs = (B + l.rows - 1) / l.rows, ncs = (D + l.chans - 1) / l.chans;
    const int64_t nslices = nrs * ncs;  // channel slices of a row slice are consecutive
    const bool split = ncs > 1;

    // three streams (in, solve, out) ordered after the work already on `stream`
    cudaStream_t sin = nullptr, scomp = nullptr, sout = nullptr;
    cudaEvent_t start = nullptr, ev_in[hp::kSlots] = {}, ev_comp[hp::kSlots] = {}, ev_out[hp::kSlots] = {};
    auto cleanup = [&]() {
        for (int k = 0; k < hp::kSlots; ++k) {
            if (ev_in[k]) cudaEventDestroy(ev_in[k]);
            if (ev_comp[k]) cudaEventDestroy(ev_comp[k]);
            if (ev_out[k]) cudaEventDestroy(ev_out[k]);
        }
        if (start) cudaEventDestroy(start);
        if (sin) cudaStreamDestroy(sin);
        if (scomp) cudaStreamDestroy(scomp);
        if (sout) cudaStreamDestroy(sout);
    };
    e = cudaStreamCreateWithFlags(&sin, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&scomp, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&sout, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&start, cudaEventDisableTiming);
    for (int k = 0; k < hp::kSlots && e == cudaSuccess; ++k) {
        e = cudaEventCreateWithFlags(&ev_in[k], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_comp[k], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_out[k], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaEventRecord(start, user);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sin, start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(scomp, start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sout, start, 0);
    if (e != cudaSuccess) {
        cudaGetLastError();
        cleanup();
        return hp::fail(PARARNN_ECUDA, "pararnn_newton_forward_host: stream or event setup failed");
    }

    const size_t row_px = (size_t)T * G * D * esz, row_h = (size_t)T * S * D * sizeof(float);
    pararnn_status st = PARARNN_OK;
    for (int64_t i = 0; i < nslices && st == PARARNN_OK; ++i) {
        const int k = (int)(i % hp::kSlots);
        const int64_t ir = i / ncs, ic = i - ir * ncs;
        const int64_t b0 = ir * l.rows, nb = (b0 + l.rows <= B) ? l.rows : B - b0;
        const int64_t d0 = ic * l.chans, dn = (d0 + l.chans <= D) ? l.chans : D - d0;
        unsigned char* slot = ws + 256 + (size_t)k * l.slot_bytes;
        void* fw = slot;
        void* px_dev = slot + hp::align256(l.fw_bytes);
        float* h_dev = reinterpret_cast<float*>(slot + hp::align256(l.fw_bytes) + l.px_bytes);
        float* w_dev = reinterpret_cast<float*>(slot + hp::align256(l.fw_bytes) + l.px_bytes + l.h_bytes);
        float* h0_dev = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(w_dev) + l.w_bytes);
        // in: the slot's pre-activations are free once the solve of slice i - kSlots is done
        if (i >= hp::kSlots) e = cudaStreamWaitEvent(sin, ev_comp[k], 0);
        const unsigned char* src = static_cast<const unsigned char*>(preacts_host) + (size_t)b0 * row_px;
        if (e == cudaSuccess && !split)
            e = cudaMemcpyAsync(px_dev, src, (size_t)nb * row_px, cudaMemcpyDefault, sin);
        if (e == cudaSuccess && split)  // nb * T * G rows of dn channels, D apart in host memory
            e = cudaMemcpy2DAsync(px_dev, (size_t)dn * esz, src + (size_t)d0 * esz, (size_t)D * esz,
                                  (size_t)dn * esz, (size_t)nb * T * G, cudaMemcpyDefault, sin);
        if (e == cudaSuccess && split && diag_w)  // (G, dn) from (G, D)
            e = cudaMemcpy2DAsync(w_dev, (size_t)dn * sizeof(float), diag_w + d0, (size_t)D * sizeof(float),
                                  (size_t)dn * sizeof(float), (size_t)G, cudaMemcpyDefault, sin);
        if (e == cudaSuccess && split && h0)  // (nb, S, dn) from (B, S, D)
            e = cudaMemcpy2DAsync(h0_dev, (size_t)dn * sizeof(float), h0 + (size_t)b0 * S * D + d0,
                                  (size_t)D * sizeof(float), (size_t)dn * sizeof(float), (size_t)nb * S,
                                  cudaMemcpyDefault, sin);
        if (e == cudaSuccess) e = cudaEventRecord(ev_in[k], sin);
        // solve: after the copy in, and after slice i - kSlots has left the slot's H
        if (e == cudaSuccess) e = cudaStreamWaitEvent(scomp, ev_in[k], 0);
        if (e == cudaSuccess && i >= hp::kSlots) e = cudaStreamWaitEvent(scomp, ev_out[k], 0);
        if (e != cudaSuccess) break;
        const float* w_use = split ? (diag_w ? w_dev : nullptr) : diag_w;
        const float* h0_use = split ? (h0 ? h0_dev : nullptr) : (h0 ? h0 + (size_t)b0 * S * D : nullptr);
        st = newton_forward_slice(B, D, cell, nb, T, dn, px_dtype, px_dev, w_use, h0_use, K, h_dev, fw, l.fw_bytes,
                                  scomp);
        if (st != PARARNN_OK) break;
        hp::fold_status<<<1, 32, 0, scomp>>>(reinterpret_cast<unsigned*>(ws), reinterpret_cast<unsigned*>(fw));
        e = cudaGetLastError();
        if (e == cudaSuccess) e = cudaEventRecord(ev_comp[k], scomp);
        // out
        if (e == cudaSuccess) e = cudaStreamWaitEvent(sout, ev_comp[k], 0);
        unsigned char* dst = reinterpret_cast<unsigned char*>(H_host) + (size_t)b0 * row_h;
        if (e == cudaSuccess && !split)
            e = cudaMemcpyAsync(dst, h_dev, (size_t)nb * row_h, cudaMemcpyDefault, sout);
        if (e == cudaSuccess && split)  // nb * T * S rows of dn channels, D apart in host memory
            e = cudaMemcpy2DAsync(dst + (size_t)d0 * sizeof(float), (size_t)D * sizeof(float), h_dev,
                                  (size_t)dn * sizeof(float), (size_t)dn * sizeof(float), (size_t)nb * T * S,
                                  cudaMemcpyDefault, sout);
        if (e == cudaSuccess) e = cudaEventRecord(ev_out[k], sout);
        if (e != cudaSuccess) break;
    }
    // `stream` continues after all three
    cudaEvent_t done[3] = {ev_in[0], ev_comp[0], ev_out[0]};
    cudaStream_t ss[3] = {sin, scomp, sout};
    for (int j = 0; j < 3 && e == cudaSuccess; ++j) {
        e = cudaEventRecord(done[j], ss[j]);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(user, done[j], 0);
    }
    cleanup();
    if (st != PARARNN_OK) return st;  // pararnn_newton_forward set the message
    if (e != cudaSuccess) {
        cudaGetLastError();
        return hp::fail(PARARNN_ECUDA, "pararnn_newton_forward_host: copy or launch failed");
    }
    return PARARNN_OK;
}

// ---- a whole training step on host buffers ----------------------------------
// The forward and the adjoint of one batch, with the pre-activations and
// dL/dH coming from host memory and H and dL/dpx going back to it, pipelined
// like the forward above but by slices of channels only: a slice holds every
// batch row of its channels, so its dL/da columns are complete sums and go
// straight to their place in dL_da.  Channels are independent recurrences and
// the tiling along T does not depend on the slice, so every value is
// bit-identical to pararnn_newton_forward + pararnn_newton_backward on the
// whole batch.

namespace pararnn {
namespace hp {

struct StepLayout {
    int64_t chans = 0;
    size_t ws_bytes = 0, px_bytes = 0, g_bytes = 0, h_bytes = 0, dpx_bytes = 0, w_bytes = 0, h0_bytes = 0,
           da_bytes = 0, slot_bytes = 0, total = 0;
};

bool step_layout(pararnn_cell cell, int64_t B, int64_t T, int64_t D, int K, int64_t channels_per_slice, size_t esz,
                 StepLayout& l) {
    const int G = pararnn_num_gates(cell), S = pararnn_state_width(cell);
    if (G < 0 || B < 0 || T < 0 || D < 0 || channels_per_slice < 0) return false;
    const bool split = channels_per_slice > 0 && channels_per_slice < D;
    if (split && (channels_per_slice % 8 != 0 || D % 8 != 0)) return false;
    l.chans = split ? channels_per_slice : (D > 0 ? D : 1);
    const int64_t Bq = B > 0 ? B : 1;
    l.ws_bytes = pararnn_workspace_bytes(cell, Bq, T, l.chans, K);
    if (l.ws_bytes == 0) return false;
    l.px_bytes = align256((size_t)Bq * T * G * l.chans * esz);
    l.g_bytes = align256((size_t)Bq * T * S * l.chans * sizeof(float));
    l.h_bytes = l.g_bytes;
    l.dpx_bytes = align256((size_t)Bq * T * G * l.chans * sizeof(float));
    l.w_bytes = align256((size_t)G * l.chans * sizeof(float));
    l.h0_bytes = align256((size_t)Bq * S * l.chans * sizeof(float));
    l.da_bytes = align256((size_t)G * l.chans * sizeof(float));
    l.slot_bytes = align256(l.ws_bytes) + l.px_bytes + l.g_bytes + l.h_bytes + l.dpx_bytes + l.w_bytes + l.h0_bytes +
                   l.da_bytes;
    l.total = 256 + kSlots * l.slot_bytes;
    return true;
}

}  // namespace hp
}  // namespace pararnn

extern "C" size_t pararnn_newton_step_host_workspace_bytes(pararnn_cell cell, int64_t B, int64_t T, int64_t D, int K,
                                                          pararnn_dtype px_dtype, int64_t channels_per_slice) {
    if (px_dtype != PARARNN_F32 && px_dtype != PARARNN_BF16) return 0;
    hp::StepLayout l;
    if (!hp::step_layout(cell, B, T, D, K, channels_per_slice, px_dtype == PARARNN_BF16 ? 2 : 4, l)) return 0;
    return l.total;
}

extern "C" pararnn_status pararnn_newton_step_host(pararnn_cell cell, int64_t B, int64_t T, int64_t D,
                                                   pararnn_dtype px_dtype, const void* preacts_host,
                                                   const float* diag_w, const float* h0, int K,
                                                   const float* dL_dH_host, float* H_host, float* dL_dpx_host,
                                                   float* dL_da, void* workspace, size_t ws_bytes,
                                                   int64_t channels_per_slice, void* stream) {
    if (px_dtype != PARARNN_F32 && px_dtype != PARARNN_BF16)
        return hp::fail(PARARNN_EINVAL, "pararnn_newton_step_host: unknown pre-activation dtype");
    const size_t esz = px_dtype == PARARNN_BF16 ? 2 : 4;
    hp::StepLayout l;
    if (!hp::step_layout(cell, B, T, D, K, channels_per_slice, esz, l))
        return hp::fail(PARARNN_EINVAL, "pararnn_newton_step_host: bad cell, sizes, K or channels_per_slice");
    if (!workspace || ws_bytes < l.total || !pointer_on_device(workspace) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255))
        return hp::fail(PARARNN_EINVAL, "pararnn_newton_step_host: workspace missing, small or not 256-byte aligned "
                                        "device memory (see pararnn_newton_step_host_workspace_bytes)");
    if ((diag_w && !pointer_on_device(diag_w)) || (h0 && !pointer_on_device(h0)) ||
        (dL_da && !pointer_on_device(dL_da)))
        return hp::fail(PARARNN_EINVAL, "pararnn_newton_step_host: diag_w, h0 and dL_da must be device memory");
    cudaStream_t user = static_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    cudaError_t e = cudaMemsetAsync(ws, 0, 256, user);
    if (e != cudaSuccess) return hp::fail(PARARNN_ECUDA, "pararnn_newton_step_host: header reset failed");
    const int G = pararnn_num_gates(cell), S = pararnn_state_width(cell);
    if (cell == PARARNN_CELL_LINEAR) dL_da = nullptr;  // no recurrent weights
    if (B == 0 || T == 0 || D == 0) {
        if (dL_da && D > 0) e = cudaMemsetAsync(dL_da, 0, sizeof(float) * G * D, user);
        return e == cudaSuccess ? PARARNN_OK : hp::fail(PARARNN_ECUDA, "pararnn_newton_step_host: dL_da reset failed");
    }
    if (!preacts_host || !dL_dH_host || !H_host || !dL_dpx_host)
        return hp::fail(PARARNN_EINVAL, "pararnn_newton_step_host: preacts, dL_dH, H and dL_dpx are required");
    // The copies out (H and dL/dpx, float32) outweigh the copies in, so the
    // pipeline runs at the pace of the copies out and only the first slice's
    // copy in is exposed: the first slice takes a quarter of the others'
    // channels (a multiple of 8), the rest channels_per_slice each.
    const int64_t first = (l.chans < D && l.chans >= 32) ? ((l.chans / 4 + 7) / 8) * 8 : l.chans;
    const int64_t ncs = 1 + (D - first + l.chans - 1) / l.chans;

    cudaStream_t sin = nullptr, scomp = nullptr, sout = nullptr;
    cudaEvent_t start = nullptr, ev_in[hp::kSlots] = {}, ev_comp[hp::kSlots] = {}, ev_out[hp::kSlots] = {};
    auto cleanup = [&]() {
        for (int k = 0; k < hp::kSlots; ++k) {
            if (ev_in[k]) cudaEventDestroy(ev_in[k]);
            if (ev_comp[k]) cudaEventDestroy(ev_comp[k]);
            if (ev_out[k]) cudaEventDestroy(ev_out[k]);
        }
        if (start) cudaEventDestroy(start);
        if (sin) cudaStreamDestroy(sin);
        if (scomp) cudaStreamDestroy(scomp);
        if (sout) cudaStreamDestroy(sout);
    };
    e = cudaStreamCreateWithFlags(&sin, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&scomp, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&sout, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&start, cudaEventDisableTiming);
    for (int k = 0; k < hp::kSlots && e == cudaSuccess; ++k) {
        e = cudaEventCreateWithFlags(&ev_in[k], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_comp[k], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_out[k], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaEventRecord(start, user);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sin, start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(scomp, start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sout, start, 0);
    if (e != cudaSuccess) {
        cudaGetLastError();
        cleanup();
        return hp::fail(PARARNN_ECUDA, "pararnn_newton_step_host: stream or event setup failed");
    }

    pararnn_status st = PARARNN_OK;
    for (int64_t ic = 0; ic < ncs && st == PARARNN_OK; ++ic) {
        const int k = (int)(ic % hp::kSlots);
        const int64_t d0 = ic == 0 ? 0 : first + (ic - 1) * l.chans;
        const int64_t want = ic == 0 ? first : l.chans;
        const int64_t dn = (d0 + want <= D) ? want : D - d0;
        unsigned char* p = ws + 256 + (size_t)k * l.slot_bytes;
        void* sws = p;
        p += hp::align256(l.ws_bytes);
        void* px_dev = p;
        p += l.px_bytes;
        float* g_dev = reinterpret_cast<float*>(p);
        p += l.g_bytes;
        float* h_dev = reinterpret_cast<float*>(p);
        p += l.h_bytes;
        float* dpx_dev = reinterpret_cast<float*>(p);
        p += l.dpx_bytes;
        float* w_dev = reinterpret_cast<float*>(p);
        p += l.w_bytes;
        float* h0_dev = reinterpret_cast<float*>(p);
        p += l.h0_bytes;
        float* da_dev = reinterpret_cast<float*>(p);
        // in: after the slot's previous slice has been solved
        if (ic >= hp::kSlots) e = cudaStreamWaitEvent(sin, ev_comp[k], 0);
        // (B*T*G rows of dn channels, D apart in host memory) and the same for dL/dH
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(px_dev, (size_t)dn * esz, static_cast<const unsigned char*>(preacts_host) + d0 * esz,
                                  (size_t)D * esz, (size_t)dn * esz, (size_t)B * T * G, cudaMemcpyDefault, sin);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(g_dev, (size_t)dn * sizeof(float), dL_dH_host + d0, (size_t)D * sizeof(float),
                                  (size_t)dn * sizeof(float), (size_t)B * T * S, cudaMemcpyDefault, sin);
        if (e == cudaSuccess && diag_w)
            e = cudaMemcpy2DAsync(w_dev, (size_t)dn * sizeof(float), diag_w + d0, (size_t)D * sizeof(float),
                                  (size_t)dn * sizeof(float), (size_t)G, cudaMemcpyDefault, sin);
        if (e == cudaSuccess && h0)
            e = cudaMemcpy2DAsync(h0_dev, (size_t)dn * sizeof(float), h0 + d0, (size_t)D * sizeof(float),
                                  (size_t)dn * sizeof(float), (size_t)B * S, cudaMemcpyDefault, sin);
        if (e == cudaSuccess) e = cudaEventRecord(ev_in[k], sin);
        // solve: after the copy in, and after the slot's previous outputs have left
        if (e == cudaSuccess) e = cudaStreamWaitEvent(scomp, ev_in[k], 0);
        if (e == cudaSuccess && ic >= hp::kSlots) e = cudaStreamWaitEvent(scomp, ev_out[k], 0);
        if (e != cudaSuccess) break;
        const float* w_use = diag_w ? w_dev : nullptr;
        const float* h0_use = h0 ? h0_dev : nullptr;
        st = newton_forward_slice(B, D, cell, B, T, dn, px_dtype, px_dev, w_use, h0_use, K, h_dev, sws, l.ws_bytes,
                                  scomp);
        if (st != PARARNN_OK) break;
        hp::fold_status<<<1, 32, 0, scomp>>>(reinterpret_cast<unsigned*>(ws), reinterpret_cast<unsigned*>(sws));
        e = cudaGetLastError();
        if (e != cudaSuccess) break;
        st = pararnn_newton_backward(cell, B, T, dn, px_dtype, px_dev, w_use, h0_use, h_dev, g_dev, dpx_dev,
                                     dL_da ? da_dev : nullptr, nullptr, sws, l.ws_bytes, scomp);
        if (st != PARARNN_OK) break;
        hp::fold_status<<<1, 32, 0, scomp>>>(reinterpret_cast<unsigned*>(ws), reinterpret_cast<unsigned*>(sws));
        e = cudaGetLastError();
        if (e == cudaSuccess && dL_da)  // (G, dn) into (G, D) at column d0
            e = cudaMemcpy2DAsync(dL_da + d0, (size_t)D * sizeof(float), da_dev, (size_t)dn * sizeof(float),
                                  (size_t)dn * sizeof(float), (size_t)G, cudaMemcpyDeviceToDevice, scomp);
        if (e == cudaSuccess) e = cudaEventRecord(ev_comp[k], scomp);
        // out
        if (e == cudaSuccess) e = cudaStreamWaitEvent(sout, ev_comp[k], 0);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(H_host + d0, (size_t)D * sizeof(float), h_dev, (size_t)dn * sizeof(float),
                                  (size_t)dn * sizeof(float), (size_t)B * T * S, cudaMemcpyDefault, sout);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(dL_dpx_host + d0, (size_t)D * sizeof(float), dpx_dev, (size_t)dn * sizeof(float),
                                  (size_t)dn * sizeof(float), (size_t)B * T * G, cudaMemcpyDefault, sout);
        if (e == cudaSuccess) e = cudaEventRecord(ev_out[k], sout);
        if (e != cudaSuccess) break;
    }
    cudaEvent_t done[3] = {ev_in[0], ev_comp[0], ev_out[0]};
    cudaStream_t ss[3] = {sin, scomp, sout};
    for (int j = 0; j < 3 && e == cudaSuccess; ++j) {
        e = cudaEventRecord(done[j], ss[j]);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(user, done[j], 0);
    }
    cleanup();
    if (st != PARARNN_OK) return st;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return hp::fail(PARARNN_ECUDA, "pararnn_newton_step_host: copy or launch failed");
    }
    return PARARNN_OK;
}
