"""Expert-cache policy oracle (test infrastructure only: the tests and the
package's smoke check may use it; the library never does).

The policy of "个人开发者用 AI 十天写出 Strata 引擎，让 12GB 显存跑起 1250 亿参数的
Qwen 3.8 Flash Next", section "命中率七成，代价是答案会变": the free GPU room holds the
experts called most often, and experts are swapped in while the conversation
runs once they start to be used frequently. The pages give no formula; the
reading used here (written out in plain Python loops, integers only):

  observe(layer, rows): on layer 0 the token clock advances by len(rows); for
      every full `epoch` of tokens every count is halved (floor). Then every
      expert id in rows adds 1 to count[layer][id].
  observe_counts(counts, tokens): the clock advances by `tokens` (halving as
      above), then counts[layer][expert] is added to every count.
  plan(slot_of, max_swaps): free slots (ascending) go to the non-resident
      (layer, expert) with count > 0 in order (count desc, layer*E+expert asc);
      then the next candidate in that order replaces the next resident in order
      (count asc, layer*E+expert desc) while its count exceeds the resident's
      by more than `margin`; at most max_swaps changes in all.
"""
from __future__ import annotations


class PolicyOracle:
    def __init__(self, L: int, E: int, S: int, epoch: int, margin: int = 0):
        self.L, self.E, self.S, self.epoch, self.margin = L, E, S, epoch, margin
        self.count = [[0] * E for _ in range(L)]
        self.clock = 0

    def observe(self, layer: int, rows) -> None:
        if layer == 0:
            self.clock += len(rows)
            while self.clock >= self.epoch:
                self.clock -= self.epoch
                for l in range(self.L):
                    for e in range(self.E):
                        self.count[l][e] //= 2
        for row in rows:
            for e in row:
                self.count[layer][int(e)] += 1

    def observe_counts(self, counts, tokens: int) -> None:
        """A window of `tokens` token steps given as counts[layer][expert]: the
        token clock advances (halving once per full epoch) before the counts are
        added -- for one token step through every layer this is observe() on
        each layer in order."""
        self.clock += tokens
        while self.clock >= self.epoch:
            self.clock -= self.epoch
            for l in range(self.L):
                for e in range(self.E):
                    self.count[l][e] //= 2
        for l in range(self.L):
            for e in range(self.E):
                self.count[l][e] += int(counts[l][e])

    def plan(self, slot_of, max_swaps: int) -> list:
        """slot_of: list of L lists of E ints (-1 = not resident), changed in place."""
        L, E = self.L, self.E
        c = lambda i: self.count[i // E][i % E]  # noqa: E731
        held = set()
        resident, candidates = [], []
        for l in range(L):
            for e in range(E):
                i = l * E + e
                if slot_of[l][e] >= 0:
                    held.add(slot_of[l][e])
                    resident.append(i)
                elif self.count[l][e] > 0:
                    candidates.append(i)
        candidates.sort(key=lambda i: (-c(i), i))
        resident.sort(key=lambda i: (c(i), -i))
        swaps = []
        ci = 0
        for s in range(self.S):
            if len(swaps) >= max_swaps or ci >= len(candidates):
                break
            if s in held:
                continue
            i = candidates[ci]
            ci += 1
            slot_of[i // E][i % E] = s
            swaps.append((s, i // E, i % E, -1, -1))
        vi = 0
        while len(swaps) < max_swaps and ci < len(candidates) and vi < len(resident):
            i, o = candidates[ci], resident[vi]
            if not c(i) > c(o) + self.margin:
                break
            s = slot_of[o // E][o % E]
            slot_of[o // E][o % E] = -1
            slot_of[i // E][i % E] = s
            swaps.append((s, i // E, i % E, o // E, o % E))
            ci += 1
            vi += 1
        return swaps
