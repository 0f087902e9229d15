"""B200-native online activation path of rotation-based W4A4 / W3A3 quantisation."""
