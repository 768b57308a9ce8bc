"""CPU oracle of the KV-aware admission scheduler (TEST INFRASTRUCTURE).

Only tests/, __graft_entry__.smoke() and bench.py's CPU baseline / reference legs may
import this module; the library's scheduler (libs3r.so, s3r_sched_simulate) shares no
code with it.

What the pages say ([News] summary: a KV-aware AIMD scheduler adapts request admission to
limit repeated KV offloading and restoring while keeping rollout parallelism, compared with
offloading at a fixed concurrency and with recomputing evicted KV, measured as pages
transferred per 1,000 generated tokens; [Explainer] Jargon, AIMD scheduler: admit one more
request when GPU KV memory has room, halve the limit under pressure; [Explainer] "Where it
earns its keep": raise concurrency while memory has room, back off when pressure or the
restore backlog grows; [Wispaper] "dense verification still needs the complete KV cache":
GPU KV utilisation measures resident pressure, the restore backlog the unmet demand of
paused requests, which keep their tokens and proposal state).

The reading taken (every step below is fixed so that two implementations agree exactly):
one iteration is one draft-and-verify round of every active request. The default backlog
mark b_high = 1 reads "too large a backlog" as more paused pages than the whole replica
holds; at half of it the cap collapses to a few requests during a long pressure event.
  1. capacity of this iteration C_t = capacity - pressure[t] pages (injected pressure).
  2. every active request, in admission order, emits min(tau[r][j], left) tokens, j its
     own round count; a request with nothing left is done and frees its pages.
  3. resident pages U = sum over active requests of ceil((prompt + generated) / 16).
  4. while U > C_t: the most recently admitted active request is evicted to the paused
     queue (FIFO): offload mode copies its pages to host memory (transferred += pages),
     recompute mode drops them.
  5. AIMD (policy "aimd"): cap = max(cap_min, cap // 2) if anything was evicted or
     U > u_high * C_t or the paused requests' pages B > b_high * C_t; else, when the cap
     binds (len(active) >= cap) and U < u_low * C_t, cap = min(cap_max, cap + 1): one more
     request when memory has room. Policy "fixed" keeps cap.
  6. admission while len(active) < cap: the head of the paused queue first (restore:
     transferred += pages in offload mode, recomputed += pages in recompute mode), else the
     next new request (prefill += its prompt pages); it must fit, U + pages <= C_t, or
     admission stops for this iteration (no skipping, so requests keep their order).
  7. time_t = c0 + c_tok * tokens_t + c_kv * U + c_xfer * transferred_t
             + c_rec * recomputed_t + c_pre * prefilled_t   (after admission, in double)
The run ends when every request is done, or after max_iters, or when an iteration can
make no progress at all (nothing active, the head of the queues does not fit): stalled.
"""
from __future__ import annotations

from collections import deque

PAGE = 16


def pages(prompt: int, generated: int) -> int:
    return -(-(prompt + generated) // PAGE)


def simulate(prompt_len, resp_len, tau, *, capacity: int, policy: str = "aimd",
             evict: str = "offload", cap0: int = 16, cap_min: int = 1, cap_max: int = 4096,
             u_low: float = 0.85, u_high: float = 0.97, b_high: float = 1.0,
             costs=(10.0, 0.0, 0.00074, 0.094, 0.5, 0.5), pressure=None, max_iters: int = 1 << 20):
    """Runs the scheduler; returns (totals dict, trace list of per-iteration tuples
    (cap, active, paused, U, transferred, recomputed, prefilled, tokens))."""
    n_req = len(prompt_len)
    prompt = [int(x) for x in prompt_len]
    resp = [int(x) for x in resp_len]
    gen = [0] * n_req
    rounds = [0] * n_req
    active: list[int] = []
    paused: deque[int] = deque()
    nxt = 0
    done = 0
    cap = cap0
    c0, c_tok, c_kv, c_xfer, c_rec, c_pre = costs
    tot = dict(tokens=0, transferred=0, recomputed=0, prefilled=0, evictions=0, time=0.0,
               iterations=0, max_active=0, stalled=0)
    trace = []
    for t in range(max_iters):
        if done == n_req:
            break
        cap_t = capacity - (int(pressure[t]) if pressure is not None and t < len(pressure) else 0)
        # 2. one round of every active request
        tokens_t = 0
        still = []
        for r in active:
            e = min(int(tau[r][rounds[r]]), resp[r] - gen[r])
            rounds[r] += 1
            gen[r] += e
            tokens_t += e
            if gen[r] >= resp[r]:
                done += 1
            else:
                still.append(r)
        active = still
        # 3. resident pages
        U = sum(pages(prompt[r], gen[r]) for r in active)
        # 4. evict the most recently admitted until it fits
        xfer = rec = pre = 0
        evicted = False
        while U > cap_t and active:
            r = active.pop()
            p = pages(prompt[r], gen[r])
            U -= p
            evicted = True
            tot["evictions"] += 1
            if evict == "offload":
                xfer += p
            paused.append(r)
        # 5. AIMD
        if policy == "aimd":
            B = sum(pages(prompt[r], gen[r]) for r in paused)
            if evicted or U > u_high * cap_t or B > b_high * cap_t:
                cap = max(cap_min, cap // 2)
            elif len(active) >= cap and U < u_low * cap_t:
                cap = min(cap_max, cap + 1)
        # 6. admission: restores first, then new requests, in order, while they fit
        while len(active) < cap:
            if paused:
                r = paused[0]
                p = pages(prompt[r], gen[r])
                if U + p > cap_t:
                    break
                paused.popleft()
                if evict == "offload":
                    xfer += p
                else:
                    rec += p
            elif nxt < n_req:
                r = nxt
                p = pages(prompt[r], 0)
                if U + p > cap_t:
                    break
                nxt += 1
                pre += p
            else:
                break
            active.append(r)
            U += p
        time_t = c0 + c_tok * tokens_t + c_kv * U + c_xfer * xfer + c_rec * rec + c_pre * pre
        tot["tokens"] += tokens_t
        tot["transferred"] += xfer
        tot["recomputed"] += rec
        tot["prefilled"] += pre
        tot["time"] += time_t
        tot["iterations"] += 1
        tot["max_active"] = max(tot["max_active"], len(active))
        trace.append((cap, len(active), len(paused), U, xfer, rec, pre, tokens_t))
        if not active and tokens_t == 0 and done < n_req and (paused or nxt < n_req) and not evicted:
            # nothing runs and nothing could be admitted: the head does not fit
            if (pressure is None or t >= len(pressure)):
                tot["stalled"] = 1
                break
    tot["done"] = done
    return tot, trace


def pages_per_1000_tokens(tot) -> float:
    return 1000.0 * tot["transferred"] / max(tot["tokens"], 1)
