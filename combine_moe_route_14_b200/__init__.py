"""B200-native MoE layer: route -> layout -> dispatch -> expert FFN -> combine."""
