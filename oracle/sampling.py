"""Seeded choice of the initial rows (TEST INFRASTRUCTURE ONLY).

The library's gmm_init picks K distinct rows of X from a seed.  This is an
independent plain-Python implementation of the two published definitions it
states, used to check it:

  SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): output i (i = 0, 1, ...) of the generator started
  at state s is mix(s + (i + 1) * 0x9E3779B97F4A7C15), where mix is the
  xor-shift / multiply finaliser with shifts 30, 27, 31 and multipliers
  0xBF58476D1CE4E5B9, 0x94D049BB133111EB.

  A uniform integer in [0, n) takes the next output x as x mod n if
  x < 2^64 - (2^64 mod n), and draws again otherwise.

  Floyd's sampling algorithm (Bentley and Floyd, "A sample of brilliance",
  CACM 1987): for j = N-K .. N-1, draw t uniform in [0, j] and take t, or j
  when t was taken already.  Every K-subset of [0, N) is equally likely; the
  k-th row is the one taken at step k.
"""
MASK = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def splitmix64(seed, i):
    """Output i of SplitMix64 started at state `seed`."""
    z = (seed + (i + 1) * GAMMA) & MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
    return z ^ (z >> 31)


class _Stream:
    def __init__(self, seed):
        self.seed = seed & MASK
        self.i = 0

    def below(self, n):
        """Uniform integer in [0, n), by rejection of the top 2^64 mod n outputs."""
        limit = (1 << 64) - ((1 << 64) % n)
        while True:
            x = splitmix64(self.seed, self.i)
            self.i += 1
            if x < limit:
                return x % n


def floyd_rows(N, K, seed):
    """K distinct row indices from [0, N) in the order Floyd's algorithm takes them."""
    if not 1 <= K <= N:
        raise ValueError("need 1 <= K <= N")
    st = _Stream(seed)
    taken, rows = set(), []
    for j in range(N - K, N):
        t = st.below(j + 1)
        v = j if t in taken else t
        taken.add(v)
        rows.append(v)
    return rows
