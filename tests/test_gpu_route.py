"""GPU parity of the uncertainty router (sparse_attn_route) against the
float64 oracle: small ragged problems and the full 128K-context workload
(28 query / 4 KV heads, 64-token blocks, 2048 query rows in 32 tiles of 64,
k = 32, rho = 2, quantile 0.25) with planted near-tie pairs."""
import pytest
import torch

import datagen as DG

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import router_harness
    return router_harness


def _small(dev, N, rows, seed):
    return DG.make_router_layer(Hq=28, Hkv=4, N=N, rows=rows, seed=seed, device=dev)


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
@pytest.mark.parametrize("N,rows,tile_rows,k,rho,q", [
    (4096, 256, 64, 8, 2, 0.25),     # 4 tiles, 2 query-vector splits per tile
    (4000, 200, 64, 8, 2, 0.5),      # ragged last tile (8 rows) and partial last block
    (2048, 96, 32, 4, 3, 0.25),      # 3 tiles, one split
    (1024, 64, 64, 16, 1, 0.25),     # rho = 1: lists are plain top-k
    (640, 128, 64, 12, 2, 1.0),      # few eligible blocks (E near k), quantile 1
    (4096, 256, 64, 8, 2, 0.0),      # quantile 0: no tile triggers, every list is trimmed to k
])
def test_route_small(cuda_dev, H, rule, N, rows, tile_rows, k, rho, q):
    lay = _small(cuda_dev, N, rows, seed=7000 + N + rows)
    kw = dict(rule=rule, block=64, q_pos0=lay.q_pos0, tile_rows=tile_rows, k=k, rho=rho, quantile=q)
    g = H.run_route_gpu(lay.k, lay.q, **kw)
    r = H.run_route_oracle(lay.k, lay.q, **kw)
    H.compare(g, r, k=k, rho=rho)
    if rho == 1:
        assert (g["kv_count"] == r.kv_count).all()


def test_route_given_tau(cuda_dev, H):
    lay = _small(cuda_dev, 4096, 256, seed=7100)
    kw = dict(rule="envelope", block=64, q_pos0=lay.q_pos0, tile_rows=64, k=8, rho=2, quantile=0.25, tau=0.3)
    g = H.run_route_gpu(lay.k, lay.q, **kw)
    r = H.run_route_oracle(lay.k, lay.q, **kw)
    assert abs(g["tau"] - 0.3) < 1e-7
    H.compare(g, r, k=8, rho=2)


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
def test_route_full_128k_planted(cuda_dev, H, rule):
    import router_plant
    lay = DG.make_router_layer(device=cuda_dev)  # 28:4, N = 131072, 2048 rows
    planted = router_plant.plant_near_ties(lay, rule=rule, block=64, tile_rows=64, k=32)
    kw = dict(rule=rule, block=64, q_pos0=lay.q_pos0, tile_rows=64, k=32, rho=2, quantile=0.25)
    g = H.run_route_gpu(lay.k, lay.q, **kw)
    r = H.run_route_oracle(lay.k, lay.q, **kw)
    st = H.compare(g, r, k=32, rho=2)
    assert len(planted) >= 0.25 * 128
    assert int(r.triggered.sum()) == 8  # 32 tiles, quantile 0.25, strict: 8 tiles below tau
    print(f"\n{rule}: planted {len(planted)} pairs, ties certified {st['ties']}, "
          f"trigger exemptions {st['trig_exempt']}, max sigma err {st['max_sigma_err']:.2e}")
