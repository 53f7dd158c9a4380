// Persistent-CTA walk over a flattened (sequence, 128-token tile) space, shared by the
// tensor-core decode kernels and the full-cache comparator.
#pragma once

#include <stdint.h>

namespace lla_walk {

// The CTAs form G / parts groups of `parts` CTAs; CTA c serves head part c % parts over the
// tile range of group c / parts, a contiguous share of the flattened (sequence, tile) space.
// The parts of a group walk the same tiles at the same time, so the LLA-2D latent row, read
// by every part, comes from L2 after its first read.  A CTA writes one record set per
// sequence it touches, with id (group + sequence) * parts + part: unique, since group and
// sequence both rise along a walk.
struct TileWalker {
    const int32_t* P;
    int B, parts;
    long long x, x1, total;
    int p, gi, b, t, nt;  // nt: tiles of sequence b (kept in a register, not re-read per tile)
    __device__ void init(const int32_t* P_, int B_, int G, int cta, int parts_) {
        P = P_;
        B = B_;
        parts = parts_;
        total = P[B];
        const int groups = G / parts;
        p = cta % parts;
        gi = cta / parts;
        x = x1 = 0;
        if (gi >= groups) return;
        x = total * gi / groups;
        x1 = total * (gi + 1) / groups;
        if (x < x1) locate();
    }
    __device__ void locate() {
        int lo = 0, hi = B - 1;  // largest b with P[b] <= x
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P[mid] <= x) lo = mid;
            else hi = mid - 1;
        }
        b = lo;
        t = int(x - P[b]);
        nt = P[b + 1] - P[b];
    }
    __device__ bool valid() const { return x < x1; }
    __device__ int key() const { return b; }  // M_q image and record set change with the sequence
    __device__ long long record_id() const { return (long long)(gi + b) * parts + p; }
    __device__ void next() {
        ++x;
        if (x >= x1) return;
        ++t;
        while (t >= nt) {
            t = 0;
            ++b;
            nt = P[b + 1] - P[b];
        }
    }
};

}  // namespace lla_walk
