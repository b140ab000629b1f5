"""Host-side study of expert placement policies over routing traces.

The pages compare, at equal cache capacity, the miss rate of their shared
routing-aware LRU with a static split that ignores routing (whole layers'
experts kept on the GPU, the layer-oriented placement they attribute to
llama.cpp's hybrid mode) and with hot-expert placement refreshed at prefill
(the behaviour they attribute to KTransformers): 16 % against 62 % of expert
reads missed for one model, 39 % against 89 % for DeepSeek-V4-Flash
("FreeToken linux", section "Rendimiento, compatibilidad y compromisos";
"FreeToken rtx 4090", section "Benchmarks, comparaciones y compromisos",
with its table of placement strategies).  This module
replays a routing trace through each policy and counts reads and misses, so
the ordering can be checked on this build's synthetic traces.

A trace is a list of calls ``(layer, expert ids)``; a read is one distinct
(layer, expert) pair of a call, the same unit the GPU cache counts.  The
policies only look at integer keys: no layer arithmetic happens here.
"""
from __future__ import annotations

import heapq

import numpy as np

Trace = list  # [(layer, np.ndarray of expert ids)]


def call_keys(layer: int, experts) -> list[tuple[int, int]]:
    """The distinct (layer, expert) reads of one call, ascending expert id."""
    return [(int(layer), int(e)) for e in np.unique(np.asarray(experts).reshape(-1))]


class SharedLru:
    """The GPU cache's policy: one LRU over (layer, expert) keys shared by all
    layers.  Per call the clock advances; hits take the new clock; each miss,
    in ascending expert order, takes the lowest free slot, else evicts the key
    with the smallest (last use, slot) that the call does not request (every
    key the call requests already carries the new clock by then)."""

    def __init__(self, capacity: int):
        self.capacity = capacity
        self.clock = 0
        self.key_of = [None] * capacity   # slot -> key
        self.stamp = [0] * capacity
        self.slot_of: dict[tuple[int, int], int] = {}
        self.free = list(range(capacity))   # min-heap of free slots
        self.lru = []                       # min-heap of (stamp, slot), stale entries skipped

    def call(self, layer: int, experts) -> tuple[int, int]:
        """-> (reads, misses) of the call; raises if it asks for more keys than slots."""
        keys = call_keys(layer, experts)
        if len(keys) > self.capacity:
            raise ValueError("call requests more distinct experts than the cache has slots")
        self.clock += 1
        t = self.clock
        misses = [k for k in keys if k not in self.slot_of]
        for k in keys:
            if k in self.slot_of:
                s = self.slot_of[k]
                self.stamp[s] = t
                heapq.heappush(self.lru, (t, s))
        for k in misses:
            if self.free:
                s = heapq.heappop(self.free)
            else:
                while True:
                    st, s = heapq.heappop(self.lru)
                    if self.key_of[s] is not None and self.stamp[s] == st and st < t:
                        break
                del self.slot_of[self.key_of[s]]
            self.key_of[s] = k
            self.slot_of[k] = s
            self.stamp[s] = t
            heapq.heappush(self.lru, (t, s))
        return len(keys), len(misses)

    def resident(self) -> dict[tuple[int, int], int]:
        """key -> slot of every resident key."""
        return dict(self.slot_of)


class StaticPlacement:
    """A fixed resident set: a read hits if its key is resident, else misses
    (the miss is served elsewhere and nothing is cached)."""

    def __init__(self, resident):
        self.resident = set(resident)

    def call(self, layer: int, experts) -> tuple[int, int]:
        keys = call_keys(layer, experts)
        return len(keys), sum(k not in self.resident for k in keys)


def layer_split(layers: int, experts: int, capacity: int) -> list[tuple[int, int]]:
    """Routing-unaware, layer-oriented placement: whole layers from layer 0 up,
    then the lowest expert ids of the next layer, until capacity keys."""
    keys = [(l, e) for l in range(layers) for e in range(experts)]
    return keys[:capacity]


def prefill_hot(prefill_trace, capacity: int) -> list[tuple[int, int]]:
    """Hot placement chosen at prefill: the `capacity` (layer, expert) keys with
    the most token assignments in the prefill routing (ties: lower layer,
    then lower expert)."""
    counts: dict[tuple[int, int], int] = {}
    for layer, experts in prefill_trace:
        for e in np.asarray(experts).reshape(-1):
            k = (int(layer), int(e))
            counts[k] = counts.get(k, 0) + 1
    order = sorted(counts, key=lambda k: (-counts[k], k[0], k[1]))
    return order[:capacity]


def replay(policy, trace) -> dict:
    """Reads, misses and miss rate of a policy over a trace."""
    reads = misses = 0
    for layer, experts in trace:
        r, m = policy.call(layer, experts)
        reads += r
        misses += m
    return {"reads": reads, "misses": misses, "miss_rate": misses / reads if reads else 0.0}


def belady(trace, capacity: int) -> dict:
    """Offline optimum for context: on a miss with the cache full, evict the
    resident key (not requested by the current call) whose next read lies
    farthest in the future.  Same read and miss counting as `replay`."""
    calls = [call_keys(layer, experts) for layer, experts in trace]
    nxt = [dict() for _ in calls]            # per call: key -> index of its next read after this call
    upcoming: dict[tuple[int, int], int] = {}
    for t in range(len(calls) - 1, -1, -1):
        for k in calls[t]:
            nxt[t][k] = upcoming.get(k, len(calls))
        for k in calls[t]:
            upcoming[k] = t
    resident: dict[tuple[int, int], int] = {}   # key -> its next read
    heap: list = []                            # (-next read, key), stale entries skipped
    reads = misses = 0
    for t, keys in enumerate(calls):
        if len(keys) > capacity:
            raise ValueError("call requests more distinct experts than the cache has slots")
        want = set(keys)
        for k in keys:
            reads += 1
            if k not in resident:
                misses += 1
                if len(resident) == capacity:
                    held = []
                    while True:
                        neg, victim = heapq.heappop(heap)
                        if resident.get(victim) != -neg:
                            continue            # stale entry
                        if victim in want:
                            held.append((neg, victim))
                            continue
                        break
                    for h in held:
                        heapq.heappush(heap, h)
                    del resident[victim]
            resident[k] = nxt[t][k]
            heapq.heappush(heap, (-nxt[t][k], k))
    return {"reads": reads, "misses": misses, "miss_rate": misses / reads if reads else 0.0}


def balanced_miss_split(misses: float, fill_bw: float, cpu_bw: float) -> float:
    """Misses to fill over the host link so that filling them takes as long as
    running the rest on the CPU: q * S / fill_bw = (m - q) * S / cpu_bw gives
    q = m * fill_bw / (fill_bw + cpu_bw).  The pages print this split garbled
    (their q exceeds m whenever the link is faster than the CPU path; "FreeToken
    290b model", section on the miss policy); this is the time-balanced reading.
    Simulated only: the library fills every miss and runs it on the GPU."""
    if misses < 0 or fill_bw <= 0 or cpu_bw <= 0:
        raise ValueError("misses must be >= 0 and bandwidths > 0")
    return misses * fill_bw / (fill_bw + cpu_bw)
