"""Plain reference of SepLLM's streaming KV cache and of one decoding step
over it.  TEST INFRASTRUCTURE ONLY: only the tests, the smoke check and the
benchmark's CPU-baseline leg use this module; it shares no code with the
CUDA path.

Sources (page title and section):
  [SEP] "SepLLM" (CSDN article), section 6.2, generation stage: the KV cache
        is split into an Initial cache (a slots), a Separator cache (s
        slots), a Local window cache (w slots) and a Past window cache that
        takes what overflows the local window; when the running size
        a + s + w + Size_past (the current contents) reaches the capacity c,
        the separators in Past move to the Separator cache and the rest of
        Past is dropped, so the running size stays within c.  Section 五,
        item 3: the average occupancy over an infinite stream is bounded by
        (w + c + a + s) / 2.
  [TALK] the talk page, section "Streaming ARMS": positions are rolled --
        the rotary positions of the cached keys are their slots in the
        cache, recomputed at every step, not their positions in the stream.

Readings (each also in the design notes):
  S1 the first a tokens of the stream fill the Initial cache; later tokens
     enter the Local window; when it holds more than w the oldest moves to
     Past;
  S2 the check "running size reaches c" happens after each append; the
     separators of Past keep their order after the separators already
     cached; if the Separator cache would hold more than s, the oldest
     separators are dropped (the page does not say which go; the oldest is
     the reading consistent with a recency-ordered cache);
  S3 the cache order (the slots) is Initial | Separator | Past | Local, the
     newest token last; a + s + w < c is required (else a full cache could
     not shrink: the page's bound (w + c + a + s)/2 < c is the same
     condition);
  S4 a decoding step is the newest token's query over every cached entry,
     with the query at slot position size - 1 and key k at position k.
"""
import numpy as np


class StreamCache:
    """Positions (stream indices) and separator flags of one sequence's cache."""

    def __init__(self, a, s, w, c):
        if not (a >= 0 and s >= 0 and w >= 1 and a + s + w < c):
            raise ValueError("need a + s + w < c")
        self.a, self.s, self.w, self.c = a, s, w, c
        self.init, self.sep, self.past, self.local = [], [], [], []  # lists of (pos, is_sep)
        self.n_seen = 0

    def size(self):
        return len(self.init) + len(self.sep) + len(self.past) + len(self.local)

    def slots(self):
        """(pos, is_sep) of every slot in cache order (S3)."""
        return self.init + self.sep + self.past + self.local

    def append(self, pos, is_sep):
        """One new token (S1, S2); returns True if the cache was compacted."""
        entry = (int(pos), bool(is_sep))
        if self.n_seen < self.a and not (self.sep or self.past or self.local):
            self.init.append(entry)
        else:
            self.local.append(entry)
            if len(self.local) > self.w:
                self.past.append(self.local.pop(0))
        self.n_seen += 1
        if self.size() >= self.c:
            kept = self.sep + [e for e in self.past if e[1]]
            self.sep = kept[max(0, len(kept) - self.s):]
            self.past = []
            return True
        return False


def decode_step(slots_k, slots_v, q, theta, rope):
    """Attention of the newest token's query q [Hq, d] over cached rows
    k, v [Hkv, n, d] with rolled positions (S4): query at n-1, key k at k.
    Returns (O [Hq, d], lse [Hq]) in float64."""
    Hkv, n, d = slots_k.shape
    Hq = q.shape[0]
    rep = Hq // Hkv
    O = np.zeros((Hq, d))
    lse = np.zeros(Hq)
    for h in range(Hq):
        g = h // rep
        qr = rope(q[h], n - 1, theta)
        z = np.array([float(qr @ rope(slots_k[g, x], x, theta)) for x in range(n)]) / np.sqrt(d)
        m = z.max()
        l = m + np.log(np.exp(z - m).sum())
        p = np.exp(z - l)
        O[h] = p @ slots_v[g]
        lse[h] = l
    return O, lse
