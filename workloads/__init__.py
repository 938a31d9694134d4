"""Seeded synthetic inputs for the equivariant convolution (graphs, features,
spherical-harmonic edge features, radial scalars).  Shared by the tests, the
oracle checks and the benchmark; holds none of the convolution's arithmetic."""
from .configs import ORDER, SPECS, Graph, Spec, edge_sh, make_graph, node_features_np, \
    node_features_torch, scalars_np, scalars_torch
from .sh import real_sh, sh_dim

__all__ = ["ORDER", "SPECS", "Graph", "Spec", "edge_sh", "make_graph", "node_features_np",
           "node_features_torch", "scalars_np", "scalars_torch", "real_sh", "sh_dim"]
