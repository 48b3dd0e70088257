"""A model of the unit-claim protocol of the tensor-core decode score pass,
on CPU: the producer's fixed first units and counter claims (one ahead), the
MMA issuer's end tiles, the two selector halves taking alternate tiles in
stretches of four, and the shared decision to leave.  Checks, for every mix
of workers, units, ring stages and tiles per unit below, that every unit is
streamed exactly once, that every worker's selectors leave because they met
an end tile (never by the loop bound), and that the first stretch's slots
stay inside its 512 keys.  Whatever order the workers' claims interleave in
(seeded shuffles) the same holds."""
import random

import pytest

import random

def run_model(nworkers, nunits, NS, KT, seed):
    rng = random.Random(seed)
    ctr = [0]
    nfixed = NS * nworkers
    # producer state per worker
    st = []
    for w in range(nworkers):
        s = {"u": 0, "c_next": 0, "c_after": 0, "units": [], "ended": False}
        if nunits > nfixed:
            s["c_next"] = ctr[0]; ctr[0] += 1
        st.append(s)
    active = list(range(nworkers))
    while active:
        w = rng.choice(active)
        s = st[w]
        u = s["u"]
        if u > nunits + NS:
            raise AssertionError("producer bound")
        if u < NS:
            unit = w + u * nworkers
        else:
            unit = nfixed + s["c_next"]
        if u == nunits + NS:
            unit = nunits
        if u >= NS and unit < nunits:
            s["c_next"] = ctr[0]; ctr[0] += 1
        s["u"] += 1
        if unit >= nunits:
            s["ended"] = True
            active.remove(w)
        else:
            s["units"].append(unit)
    seen = sorted(x for s in st for x in s["units"])
    assert seen == list(range(nunits)), (seen[:10], nunits)
    # per worker: tiles and selectors
    max_stretch = (nunits * KT + 2 + 3) // 4
    for s in st:
        tiles = []
        for unit in s["units"]:
            for q in range(KT):
                tiles.append(unit * KT * 128 + q * 128)
        tiles += [-1, -1]
        done = [False, False]
        ended = False
        m = 0
        first_tiles = 0
        while True:
            for half in (0, 1):
                t = m * 4 + half
                while t < (m + 1) * 4 and not done[half]:
                    assert t < len(tiles), "selector waits for a tile never produced"
                    if tiles[t] < 0:
                        done[half] = True; ended = True; break
                    if m == 0:
                        first_tiles = max(first_tiles, t + 1)
                        assert t * 128 + 127 < 512
                    t += 2
            last = m >= max_stretch
            if last or ended:
                assert ended, "stopped by the bound"
                break
            m += 1
        assert first_tiles == min(len(tiles) - 2, 4)
    return True



@pytest.mark.parametrize("KT", [1, 2])
@pytest.mark.parametrize("NS", [2, 3, 4])
def test_claim_protocol(NS, KT):
    for nworkers in (1, 2, 3, 5, 36, 37, 74):
        for nunits in (0, 1, 2, 3, 7, 35, 36, 37, 100, 145, 1024):
            for seed in range(5):
                run_model(nworkers, nunits, NS, KT, seed)
