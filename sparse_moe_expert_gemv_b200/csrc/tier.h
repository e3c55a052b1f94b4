// tier.h -- replacement policy of the HBM expert-slot cache when the
// experts' backing copies live in host memory (host code only, no CUDA).
//
// The Strata engine analysis article ("93 token/s on one 8 GB card",
// section "Expert cache") keeps the hot experts of a model larger than the
// GPU's memory in a fixed set of device slots: a (layer, expert) either has a
// slot or is a miss, and misses are brought in while other work runs.  The
// user report "EPYC 7B13 + 2x RTX 3090" raises the hit rate from 92.7 % to
// 99.2 % by making the cache adaptive instead of static.  Here a window's
// routing (the experts it selects) is a request set; every selected expert
// without a slot takes one, evicting the expert with the lowest score among
// those the current request does not need:
//   kLru       score = the last call that used it (least recently used);
//   kAdaptive  score = the expert's exponentially decayed use count
//              (half-life of `half_life` requests), ties broken by recency.
//              The count is kept per (layer, expert), resident or not, so an
//              expert that many recent windows chose keeps its history across
//              an eviction and outlives a burst of experts used once.
#pragma once

#include <cmath>
#include <cstdint>
#include <vector>

namespace moe {

enum TierPolicy { kLru = 0, kAdaptive = 1 };

struct TierCache {
  int n_slots = 0, policy = kLru;
  double half_life = 64.0;
  long long now = 0;                 // calls so far
  std::vector<long long> owner;      // [n_slots] key (layer * E + expert) or -1
  std::vector<long long> last_use;   // [n_slots] request of the slot's last use
  std::vector<long long> stamp;      // [n_slots] request that last pinned the slot
  std::vector<double> kscore;        // [n_keys] decayed use count at klast
  std::vector<long long> klast;      // [n_keys] request of the key's last use (-1: never)
  long long hits = 0, misses = 0, evictions = 0;

  void init(int slots, int pol, double hl, long long n_keys) {
    n_slots = slots;
    policy = pol;
    half_life = hl > 0 ? hl : 64.0;
    now = 0;
    owner.assign(slots, -1);
    last_use.assign(slots, -1);
    stamp.assign(slots, -1);
    kscore.assign((size_t)n_keys, 0.0);
    klast.assign((size_t)n_keys, -1);
    hits = misses = evictions = 0;
  }

  // decayed use count of key k as of request `now`
  double decayed(long long k) const {
    if (klast[(size_t)k] < 0) return 0.0;
    return kscore[(size_t)k] * std::exp2(-(double)(now - klast[(size_t)k]) / half_life);
  }

  // this request uses key k, held in slot s
  void touch(int s, long long k) {
    kscore[(size_t)k] = decayed(k) + 1.0;
    klast[(size_t)k] = now;
    last_use[s] = now;
    stamp[s] = now;
  }

  // One request: the distinct keys of a window (slot_of maps a key to its
  // slot or -1, and is updated).  For each key that had to be brought in,
  // (key, slot, evicted key or -1) is appended to the fill lists.  With
  // protect_prev, the slots of the previous request are not evicted either
  // (its window may still be running while this one is prefetched).
  // Returns false, changing nothing but the hits' use counts, when the
  // misses outnumber the slots that may be taken.
  bool request(const std::vector<long long> &keys, std::vector<int> &slot_of, bool protect_prev,
               std::vector<long long> &fill_key, std::vector<int> &fill_slot,
               std::vector<long long> &fill_evicted) {
    ++now;
    // pin the hits first, so no miss evicts an expert this window uses
    int n_miss = 0;
    for (long long k : keys) {
      const int s = slot_of[(size_t)k];
      if (s >= 0)
        touch(s, k);
      else
        ++n_miss;
    }
    int avail = 0;
    for (int s = 0; s < n_slots; ++s)
      if (stamp[s] != now && !(protect_prev && stamp[s] == now - 1)) ++avail;
    if (n_miss > avail) return false;
    hits += (long long)keys.size() - n_miss;
    for (long long k : keys) {
      if (slot_of[(size_t)k] >= 0) continue;
      ++misses;
      int best = -1;
      double best_score = 0.0;
      long long best_last = 0;
      for (int s = 0; s < n_slots; ++s) {
        if (stamp[s] == now || (protect_prev && stamp[s] == now - 1)) continue;
        if (owner[s] < 0) {  // a free slot wins at once
          best = s;
          break;
        }
        const double sc = policy == kLru ? (double)last_use[s] : decayed(owner[s]);
        if (best < 0 || sc < best_score || (sc == best_score && last_use[s] < best_last)) {
          best = s;
          best_score = sc;
          best_last = last_use[s];
        }
      }
      const long long ev = owner[best];
      if (ev >= 0) {
        slot_of[(size_t)ev] = -1;
        ++evictions;
      }
      owner[best] = k;
      slot_of[(size_t)k] = best;
      touch(best, k);
      fill_key.push_back(k);
      fill_slot.push_back(best);
      fill_evicted.push_back(ev);
    }
    return true;
  }

  // Rebuild the owners from a slot table set wholesale.
  void adopt(const std::vector<int> &slot_of) {
    owner.assign(n_slots, -1);
    for (size_t key = 0; key < slot_of.size(); ++key)
      if (slot_of[key] >= 0 && slot_of[key] < n_slots) owner[slot_of[key]] = (long long)key;
  }
};

}  // namespace moe
