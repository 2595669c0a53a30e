// decode_wl.cuh -- the one-token work list, written by a single warp of the
// router or plan kernel right after it knows the token's slots and gate
// weights: entry 0 is the shared expert (if any), then one entry per k in k
// order (a token's slots are distinct).  Same layout the work-list builder
// produces, with the O(1) unit map fields of WorkList filled in.
#pragma once
#include "common.cuh"

namespace moe {

// lane k < K holds slot and gate weight of selection k and `take` (whether
// selection k belongs to this list); all 32 lanes call.  The taken selections
// become entries nsh, nsh+1, ... in k order; their h rows stay at k*F.
__device__ __forceinline__ void write_decode_worklist(const DecodeWLTarget& t, int K, int slot, float w, bool take) {
    const int lane = threadIdx.x & 31;
    const int nsh = t.shared_blob ? 1 : 0;
    const int nsg = t.D / kGuSlice, tiles = t.D / kChunkRows;
    const int ush = t.shared_blob ? (t.FS / 16) * nsg : 1, urt = (t.F / 16) * nsg;
    const int ns_sh = t.shared_blob ? t.FS / down_ks(t.FS) : 1, ns_rt = t.F / down_ks(t.F);
    const bool mine = lane < K && take;
    const uint32_t ball = __ballot_sync(0xffffffffu, mine);
    const int nr = __popc(ball);
    if (mine) {
        const int j = __popc(ball & ((1u << lane) - 1u));  // rank among the taken selections
        const int e = nsh + j;
        FfnEntry en;
        en.blob = t.slot_base + size_t(slot) * t.slot_stride;
        en.ready = t.ready ? t.ready + slot : nullptr;
        en.ready_val = t.ready_val;
        en.F = t.F;
        en.n_rows = 1;
        en.row0 = e;
        en.ubase_gu = nsh * ush + j * urt;
        en.ubase_dn = tiles * (nsh * ns_sh + j * ns_rt);
        t.entries[e] = en;
        FfnRow r;
        r.x_row = 0;
        r.h_off = lane * t.F;
        r.y_row = 0;
        r.w = w;
        t.rows[e] = r;
    }
    if (lane == 0) {
        if (nsh) {
            FfnEntry en;
            en.blob = t.shared_blob;
            en.ready = nullptr;
            en.ready_val = 0;
            en.F = t.FS;
            en.n_rows = 1;
            en.row0 = 0;
            en.ubase_gu = 0;
            en.ubase_dn = 0;
            t.entries[0] = en;
            FfnRow r;
            r.x_row = 0;
            r.h_off = t.h_shared_off;
            r.y_row = 0;
            r.w = 1.0f;
            t.rows[0] = r;
        }
        WorkList wl;
        wl.n_entries = nsh + nr;
        wl.units_gu = nsh * ush + nr * urt;
        wl.units_per_tile_dn = nsh * ns_sh + nr * ns_rt;
        wl.units_dn = tiles * wl.units_per_tile_dn;
        wl.T = 1;
        wl.max_rows = 1;
        wl.n_shared = nsh;
        wl.ush_gu = ush;
        wl.urt_gu = urt;
        wl.ns_sh_dn = ns_sh;
        wl.ns_rt_dn = ns_rt;
        wl.F = t.F;
        wl.FS = t.FS;
        *t.wl = wl;
    }
}

}  // namespace moe
