"""Seeded synthetic inputs for the equivariant convolution (graphs and edge vectors,
node features, drawn edge scalars, radial-MLP weights).  Shared by the tests, the
oracle checks and the benchmark; holds none of the method's arithmetic (the
harmonics and the radial MLP are evaluated by each side from the edge vectors)."""
from .configs import ORDER, SPECS, Graph, Spec, edge_vectors_np, make_graph, node_features_np, \
    node_features_torch, radial_weights, scalars_np, scalars_torch

__all__ = ["ORDER", "SPECS", "Graph", "Spec", "edge_vectors_np", "make_graph",
           "node_features_np", "node_features_torch", "radial_weights", "scalars_np",
           "scalars_torch"]
