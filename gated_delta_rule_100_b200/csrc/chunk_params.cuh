// chunk_params.cuh -- launch parameters of the prefill kernels, shared by the
// kernels (prep_fwd.cu, exact_prep.cu, chain_fwd.cu) and the C ABI
// (kda_api.cu), and the token geometry they decode their work from.
#pragma once
#include <stdint.h>

#include "chunk_common.cuh"
#include "kda_device.cuh"

namespace kda {

// Token geometry of one prefill launch.
//
// Uniform (cu == NULL): B = nseqs sequences of T tokens in the [B, T, H, *]
// layout; the launch covers local chunks [n_begin, n_begin + nseg) of every
// sequence.  Item (b H + h) nseg + (chunk - n_begin) is also its record index.
//
// Packed (cu != NULL): nseqs sequences concatenated along the token axis
// ([T_total, H, *], T = T_total); sequence n holds tokens cu[n] .. cu[n+1] - 1
// and global chunks cc[n] .. cc[n+1] - 1 (a chunk never crosses a sequence
// boundary; the last chunk of a sequence may be partial).  The launch covers
// the window of global chunks [c0, c0 + W) of every head: item
// (chunk - c0) H + h, record h W + (chunk - c0), so the records of one
// (sequence, head) are consecutive.
struct SeqGeom {
    const int *cu;         // [nseqs + 1] token offsets (checked by the setup kernel), or NULL
    const int *cc;         // [nseqs + 1] chunk offsets (packed)
    const int *chunk_seq;  // sequence of every global chunk (packed)
    int nseqs;             // sequences: B (uniform) or N (packed)
    int T;                 // tokens per sequence (uniform) or in all (packed)
    int n_begin, nseg;     // uniform: the segment of local chunks
    int c0, W;             // packed: the window of global chunks
};

// Where one prep item (one chunk of one head) lives.
struct ItemGeo {
    int h, seq;
    int tok0, bcoord;   // coordinates of its first token in the q/k tensor maps (token, batch)
    long long row0;     // flattened token row of its first token (b T + t0, or cu[n] + t0)
    int nvalid;         // tokens of its sequence from the first on; later rows are padding
    long long rec;      // record index
};

__device__ __forceinline__ bool geom_packed(const SeqGeom &gm) { return gm.cu != nullptr; }

// Token rows of the launch's tensors ([rows, H, *]).
__device__ __forceinline__ long long geom_rows(const SeqGeom &gm) {
    return geom_packed(gm) ? (long long)gm.T : (long long)gm.nseqs * gm.T;
}

// Items of the launch (packed: read from the device-side chunk offsets).
// PACKED: the launch's geometry form, known at compile time (kernels that take
// both forms pass the runtime test).
template <bool PACKED>
__device__ __forceinline__ int geom_items(const SeqGeom &gm, int H) {
    if (!PACKED) return gm.nseqs * H * gm.nseg;
    const int left = gm.cc[gm.nseqs] - gm.c0;
    return (left < gm.W ? (left > 0 ? left : 0) : gm.W) * H;
}

template <bool PACKED>
__device__ __forceinline__ ItemGeo item_geo(const SeqGeom &gm, int H, int it) {
    ItemGeo r;
    if (!PACKED) {
        const int ni = it % gm.nseg, bh = it / gm.nseg;
        r.h = bh % H;
        r.seq = bh / H;
        const int t0 = (gm.n_begin + ni) * CH;
        r.tok0 = t0;
        r.bcoord = r.seq;
        r.row0 = (long long)r.seq * gm.T + t0;
        r.nvalid = gm.T - t0;
        r.rec = it;
    } else {
        const int lc = it / H;  // chunk - c0
        r.h = it % H;
        const int ci = gm.c0 + lc;
        const int n = gm.chunk_seq[ci];
        const int t0 = (ci - gm.cc[n]) * CH;
        r.seq = n;
        r.row0 = (long long)gm.cu[n] + t0;
        r.tok0 = (int)r.row0;
        r.bcoord = 0;
        r.nvalid = gm.cu[n + 1] - gm.cu[n] - t0;
        r.rec = (long long)r.h * gm.W + lc;
    }
    return r;
}

// The chunks one chain CTA (sequence seq, head h) walks in this launch.
struct ChainGeo {
    long long row0;   // flattened token row of the sequence's first token
    int len;          // tokens of the sequence
    int lc0, nch;     // first local chunk, chunks in this launch
    long long rec0;   // record index of the first of them
    bool first, last; // the launch holds the sequence's first / last chunk (the state's start / end)
};

// Uniform launches may split the segment into `parts` parts of part_len chunks
// (the two-level pass); packed launches have one part.
__device__ __forceinline__ ChainGeo chain_geo(const SeqGeom &gm, int H, int seq, int h, int part = 0,
                                              int parts = 1, int part_len = 0) {
    ChainGeo r;
    if (!geom_packed(gm)) {
        const int off = part * part_len;
        const int left = gm.nseg - off;
        r.row0 = (long long)seq * gm.T;
        r.len = gm.T;
        r.lc0 = gm.n_begin + off;
        r.nch = parts == 1 ? gm.nseg : (left < part_len ? (left > 0 ? left : 0) : part_len);
        r.rec0 = (long long)(seq * H + h) * gm.nseg + off;
        r.first = gm.n_begin == 0 && part == 0;
        r.last = (gm.n_begin + gm.nseg) * CH >= gm.T && part == parts - 1;
    } else {
        const int a = gm.cc[seq], e = gm.cc[seq + 1];
        const int lo = a > gm.c0 ? a : gm.c0;
        const int hi = e < gm.c0 + gm.W ? e : gm.c0 + gm.W;
        r.row0 = gm.cu[seq];
        r.len = gm.cu[seq + 1] - gm.cu[seq];
        r.lc0 = lo - a;
        r.nch = hi > lo ? hi - lo : 0;
        r.rec0 = (long long)h * gm.W + (lo - gm.c0);
        if (a == e) {  // an empty sequence: its state passes through in the first window
            r.first = r.last = gm.c0 == 0;
        } else {
            r.first = r.nch > 0 && lo == a;
            r.last = r.nch > 0 && hi == e;
        }
    }
    return r;
}

// Items of a launch, claimed by persistent CTAs (see SeqGeom).
struct PrepParams {
    const float *g;      // gate [tokens, H, g_dk]
    int g_dk;            // gate values per (token, head): dk (per key channel) or 1 (one, broadcast)
    const float *beta;   // [tokens, H]
    uint8_t *ws;         // records, REC_BYTES each, at their record index
    long long nrec;      // records in ws (the debug build checks record indices against it)
    int *ticket;         // item counter, zero at launch: CTAs claim items from it
    int *steep_count;    // zero at launch: items appended to steep_items
    int *steep_items;    // items whose decay needs the exact kernel (room for every item)
    int force_exact;     // test hook: list every item
    int block_refs;      // test hook: the 16-token block references for every item, mild or not
    float gate_c;        // gate prologue (raw g, beta, q, k): g = -gate_c softplus(g_raw)
    int H;
    SeqGeom gm;
    DeviceStatus st;
    unsigned long long *stamp;  // measurement hook: this launch's timing slot, or NULL
};

// The exact kernel (exact_prep.cu): rewrites P, T' and W of the listed items.
struct ExactParams {
    const uint16_t *q, *k;  // bf16 [tokens, H, dk]
    const float *g;         // [tokens, H, g_dk]
    int g_dk;
    const float *beta;      // [tokens, H]
    uint8_t *ws;            // records, as in PrepParams
    long long nrec;
    const int *steep_count, *steep_items;
    int prologue;           // raw g, beta, q, k: apply the gate prologue and normalise q, k
    float gate_c;
    int H;
    SeqGeom gm;
    DeviceStatus st;
    unsigned long long *stamp;
};

// One CTA per (sequence, head, part, slot); walks its chunks of the launch in order.
//
// Two-level pass (uniform path, few (b, h), long segments): the segment's chunks
// are cut into `parts` parts of part_len chunks.  Pass A (pass_a != 0) covers
// parts 0 .. parts - 2: part 0 runs as usual from the segment's start state and
// writes its end state to p_start[1]; every other part runs as a "transition":
// value slots start from a zero state and write their end state to p_local[p],
// identity slots carry the columns of the dk x dk identity instead of values
// (V = 0) and write p_trans[p]; transitions write no outputs.  Then
// p_start[p + 1] = p_trans[p] p_start[p] + p_local[p] (parts_fixup.cu), and
// pass B runs parts 1 .. parts - 1 from p_start[p] with outputs, the last part
// writing the segment's end state.  parts == 1: the plain pass.
struct ChainParams {
    const uint16_t *v;   // bf16 [tokens, H, dv]
    const float *h0;     // [nseqs, H, dk, dv] or NULL: the state before the sequence's first chunk
    uint16_t *out;       // bf16 [tokens, H, dv]
    float *hT;           // [nseqs, H, dk, dv] or NULL: the state after the sequence's last chunk
    float *carry;        // packed: [nseqs, H, dk, dv], the state between windows (may be hT)
    const uint8_t *ws;   // records written by the prep kernel
    long long nrec;      // records in ws (tensor-map extent)
    float scale;
    int H, DV, nslices;
    int parts, part_len;  // the segment's parts (1: the plain pass)
    int part0, nparts;    // parts in this launch
    int slots;            // CTAs per (sequence, head, part): value slices, plus identity slices in pass A
    int pass_a;
    float *p_start, *p_local, *p_trans;  // [parts][nseqs H][dk][dv | dv | dk]
    SeqGeom gm;
    DeviceStatus st;
    uint64_t inject_wait_polls;  // test hook: nonzero = first wait on a barrier nothing signals
    unsigned long long *stamp;
};

}  // namespace kda
