// Dispatch order of the backward's grid (one CTA per sequence, KV head and 128-key
// tile). Host code only: no CUDA types, so the rule can be checked on any machine.
#pragma once

namespace fa {

// True when the key tiles of one (sequence, KV head) are to be dispatched next to each
// other (key tile fastest in the grid); false when a masked grid dispatches the first
// key tiles, which see the most query tiles, first (key tile slowest). Without a mask
// every key tile of a head walks all its query tiles and the grid is key tile fastest
// either way.
//
// With d = 128 and one query head per KV head (walks a quarter as long as under 4-way
// grouping), key-tile-first lets neighbouring CTAs read the same Q and dO tiles and
// reduce into the same dQ lines (B=1 N=4096 Hq=Hkv=32: DRAM reads 202 against 447 MB,
// reduction hit rate 63 against 55 %). It pays once the grid holds enough waves that each
// head's longest walk starting late does not make the tail (Hq = Hkv = 32, causal,
// TFLOP/s key-tile-first against heaviest first: 512 CTAs 469 / 552, 1024 CTAs 658-664 /
// 661-689, 2048 CTAs 575-766 / 529-732, 4096 CTAs 761-765 / 676-677). With 4-way grouping
// heaviest first is faster (785 against 767). Anchor keys keep heaviest first: the tile
// holding them is walked by every query tile, and started late it becomes the tail
// (window of 1024 + 4 anchors, Hq = Hkv = 32: 487 against 460 TFLOP/s; the plain window
// runs at 585 in either order).
inline bool bwd_key_tile_fastest(bool masked, int d, int Hq, int Hkv, int n_anchor, long long n_ctas, int sms) {
    return masked && d == 128 && Hq == Hkv && n_anchor == 0 && n_ctas >= 12LL * sms;
}

}  // namespace fa
